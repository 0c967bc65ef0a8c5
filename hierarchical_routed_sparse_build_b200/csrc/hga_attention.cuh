// Exact softmax attention of the R <= 8 query heads of one KV head over a routed
// token list, one warp per 16-token tile, bf16 tensor-core MMAs with fp32
// accumulation and an online (running-max) softmax.
//
// "Hierarchical Global Attention (HGA)", abstract: attention over the routed
// tokens is exact; only the token set is approximate. The R query heads that
// share a KV head use every K/V tile once (GQA head sharing), which turns the
// per-tile work into two small dense products:
//
//   S^T[16 tok x 8 heads]  = K_tile[16 x D] . Q^T[D x 8]        (mma m16n8k16, D/16 k-steps)
//   O^T[D x 8 heads]      += V_tile^T[D x 16] . P^T[16 x 8]     (mma m16n8k16, D/16 m-tiles)
//
// Tokens are the MMA rows, heads the 8 columns, so no MMA work is padded.
//
// Register-direct gather. Each K/V byte of a routed tile is used by exactly one
// MMA, so tiles go straight from HBM into the fragment registers with 16-byte
// loads; there is no shared-memory staging and no reuse to exploit. Both
// contractions run over an index (head dim for QK^T, tokens for PV) whose order
// is free, and so is the order of the output rows of O^T. The kernels use that
// freedom to make every thread's fragment a set of whole 16-byte runs of one
// key/value row:
//
//   K: lane (g, t) [g = lane/4, t = lane%4] loads rows g and g+8 of the tile at
//      columns 8t + 32j .. +7 (j < D/32). For k-step s = 2j+p the A fragment is
//      words 2p and 2p+1 of load j, so logical k = 2t+dl maps to column
//      8t + 32j + 4p + dl and k = 2t+8+dl to 8t + 32j + 4p + 2 + dl. The Q^T (B)
//      fragment uses the same map; it is staged once per CTA in shared memory.
//   V: lane (g, t) loads rows 2t, 2t+1, 2t+8, 2t+9 (the PV k index) at columns
//      8g + 64h .. +7 (h < D/64). m-tile mt takes word w = mt%4 of load
//      h = mt/4; its low half is output row d(mt, g) = 8g + 64h + 2w and its
//      high half is row g+8 = d(mt, g) + 1. prmt pairs two tokens per register.
//   P: the S^T accumulator holds (tokens g, g+8) x (heads 2t, 2t+1); the PV B
//      fragment needs (tokens 2t.., 2t+8..) x (head g): one movmatrix.trans per
//      8x8 half converts it in registers.
//
// A warp's loads per tile: 8 + 8 x 16 B per lane for D = 128, each instruction
// covering whole 32-byte sectors. The next tile's loads are issued before the
// current tile's math (register double buffering).
#pragma once

#include "hga_common.cuh"

namespace hga {

template <int D>
struct AttnTile {
  static constexpr int KJ = D / 32;  // 16-byte K loads per row per lane
  static constexpr int VH = D / 64;  // 16-byte V loads per row per lane
  uint4 ka[KJ], kb[KJ];              // K rows g, g+8
  uint4 va[4][VH];                   // V rows 2t, 2t+1, 2t+8, 2t+9
  int n_valid;                       // entries 0 .. n_valid-1 of the tile are real tokens
};

// Q^T (B operand) fragments of all k-steps, shared by the warps of a CTA (they
// attend with the same heads): load j of lane l is qfrag[j * 32 + l], words
// {x, y} feeding k-step 2j and {z, w} k-step 2j+1. Lanes read consecutive
// 16-byte slots, so the shared-memory reads are conflict-free.
template <int D>
__device__ __forceinline__ void stage_q_fragments(uint4* qfrag, const uint16_t* q_heads, int R,
                                                  int tid, int nthreads) {
  for (int i = tid; i < (D / 32) * 32; i += nthreads) {
    const int j = i >> 5, l = i & 31, g = l >> 2, t = l & 3;
    qfrag[i] = g < R ? ldg_nc(q_heads + (int64_t)g * D + 8 * t + 32 * j) : make_uint4(0, 0, 0, 0);
  }
}

template <int D>
struct AttnState {
  static constexpr int MT = D / 16;  // PV m-tiles
  float o[MT][4];                    // O^T accumulators: rows d(mt,g), d(mt,g)+1 x heads 2t, 2t+1
  float m0, m1;                      // running max (log2 units) of heads 2t, 2t+1
  float l0, l1;                      // running denominators (lane-partial)

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[mt][i] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  }
};

// Load tile rows[0..15] (row indices in head_dim units). Every entry holds a
// readable row: entries at or past n_valid repeat a real row of the batch and
// are masked out in compute_tile, so the loads need no predicate.
template <int D>
__device__ __forceinline__ void load_tile(AttnTile<D>& T, const uint32_t* rows, int n_valid,
                                          const uint16_t* K, const uint16_t* V, int lane) {
  const int g = lane >> 2, t = lane & 3;
  T.n_valid = n_valid;
  const uint16_t* k0 = K + (int64_t)rows[g] * D + 8 * t;
  const uint16_t* k1 = K + (int64_t)rows[g + 8] * D + 8 * t;
#pragma unroll
  for (int j = 0; j < AttnTile<D>::KJ; ++j) {
    T.ka[j] = ldg_stream(k0 + 32 * j);
    T.kb[j] = ldg_stream(k1 + 32 * j);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int entry = 2 * t + (i & 1) + 8 * (i >> 1);
    const uint16_t* vp = V + (int64_t)rows[entry] * D + 8 * g;
#pragma unroll
    for (int h = 0; h < AttnTile<D>::VH; ++h) T.va[i][h] = ldg_stream(vp + 64 * h);
  }
}

// One tile: S^T = K Q^T, online softmax, O^T += V^T P^T. sl = scale * log2(e).
template <int D>
__device__ __forceinline__ void compute_tile(AttnState<D>& st, const AttnTile<D>& T,
                                             const uint4* qfrag, float sl, int lane) {
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < D / 32; ++j) {
    const uint4 qv = qfrag[j * 32 + lane];
    mma_16816(s, T.ka[j].x, T.kb[j].x, T.ka[j].y, T.kb[j].y, qv.x, qv.y);
    mma_16816(s, T.ka[j].z, T.kb[j].z, T.ka[j].w, T.kb[j].w, qv.z, qv.w);
  }
  // s[0]: token g, head 2t   s[1]: token g, head 2t+1
  // s[2]: token g+8, head 2t s[3]: token g+8, head 2t+1
  {
    const int g = lane >> 2;
    if (g >= T.n_valid) s[0] = s[1] = -INFINITY;
    if (g + 8 >= T.n_valid) s[2] = s[3] = -INFINITY;
  }
  float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, off));
  }
  const float mn0 = fmaxf(st.m0, mx0 * sl), mn1 = fmaxf(st.m1, mx1 * sl);
  const float base0 = mn0 == -INFINITY ? 0.f : mn0;
  const float base1 = mn1 == -INFINITY ? 0.f : mn1;
  const float alpha0 = ex2(st.m0 - base0), alpha1 = ex2(st.m1 - base1);
  const float p0 = ex2(fmaf(s[0], sl, -base0)), p1 = ex2(fmaf(s[1], sl, -base1));
  const float p2 = ex2(fmaf(s[2], sl, -base0)), p3 = ex2(fmaf(s[3], sl, -base1));
  st.l0 = fmaf(st.l0, alpha0, p0 + p2);
  st.l1 = fmaf(st.l1, alpha1, p1 + p3);
  st.m0 = mn0;
  st.m1 = mn1;
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    st.o[mt][0] *= alpha0;
    st.o[mt][1] *= alpha1;
    st.o[mt][2] *= alpha0;
    st.o[mt][3] *= alpha1;
  }
  // P^T halves (tokens 0-7, 8-15) -> PV B fragments (head g, tokens 2t.. / 2t+8..)
  const uint32_t b0 = movmatrix_trans(pack_bf16x2(p0, p1));
  const uint32_t b1 = movmatrix_trans(pack_bf16x2(p2, p3));
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    const int h = mt >> 2, w = mt & 3;
    const uint32_t x0 = word_of(T.va[0][h], w), x1 = word_of(T.va[1][h], w);
    const uint32_t x2 = word_of(T.va[2][h], w), x3 = word_of(T.va[3][h], w);
    mma_16816(st.o[mt], prmt(x0, x1, 0x5410), prmt(x0, x1, 0x7632), prmt(x2, x3, 0x5410),
              prmt(x2, x3, 0x7632), b0, b1);
  }
}

// Output row of O^T held in low accumulators of m-tile mt by lanes with this g.
__host__ __device__ constexpr int o_row(int mt, int g) { return 8 * g + 64 * (mt >> 2) + 2 * (mt & 3); }

// Warp over the tiles tile0, tile0+stride, ... < n_tiles of a staged row table
// holding n_entries real entries. Two tile buffers alternate so that the next
// tile's loads are in flight during the current tile's math.
template <int D>
__device__ __forceinline__ void attend_tiles(AttnState<D>& st, const uint32_t* rows, int n_entries,
                                             int tile0, int stride, const uint16_t* K,
                                             const uint16_t* V, const uint4* qfrag, float sl,
                                             int lane) {
  const int n_tiles = (n_entries + 15) >> 4;
  int tile = tile0;
  if (tile >= n_tiles) return;
  AttnTile<D> A, B;
  load_tile<D>(A, rows + 16 * tile, n_entries - 16 * tile, K, V, lane);
  while (true) {
    const int t1 = tile + stride;
    if (t1 < n_tiles) load_tile<D>(B, rows + 16 * t1, n_entries - 16 * t1, K, V, lane);
    compute_tile<D>(st, A, qfrag, sl, lane);
    if (t1 >= n_tiles) break;
    const int t2 = t1 + stride;
    if (t2 < n_tiles) load_tile<D>(A, rows + 16 * t2, n_entries - 16 * t2, K, V, lane);
    compute_tile<D>(st, B, qfrag, sl, lane);
    if (t2 >= n_tiles) break;
    tile = t2;
  }
}

}  // namespace hga
