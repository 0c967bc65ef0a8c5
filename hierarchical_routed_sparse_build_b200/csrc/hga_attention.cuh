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
// Tokens are the MMA rows and heads the 8 columns, so no MMA work is padded.
//
// Data path of one tile (per warp, no CTA barrier):
//   1. HBM -> registers: coalesced 16-byte loads, each warp instruction reading
//      whole key/value rows (D*2 bytes per row, 512 contiguous bytes for D = 128).
//      The next tile's loads are issued before the current tile's math.
//   2. registers -> a warp-private shared tile, swizzled (below); K and V of a
//      tile pass through the same 16-row buffer one after the other, keeping
//      shared memory small (L1 keeps the rest of the SM's 256 KB for the
//      return data of loads in flight).
//   3. shared tile -> MMA fragments. Both contractions run over an index whose
//      order is free (head dim for QK^T, tokens for PV), and so is the order of
//      the O^T rows; the fragment maps below make every fragment a set of whole
//      16-byte units of one row:
//        K: lane (g, t) [g = lane/4, t = lane%4] takes rows g and g+8, units
//           t + 4j (j < D/32). k-step 2j+p uses words 2p, 2p+1 of unit j, so
//           logical k = 2t+dl is column 8t + 32j + 4p + dl and k = 2t+8+dl is
//           8t + 32j + 4p + 2 + dl; the Q^T (B) fragment uses the same map.
//        V: lane (g, t) takes rows 2t, 2t+1, 2t+8, 2t+9 (the PV k index) at
//           units vu(g, h) = 8h + 4(g&1) + g/2 (h < D/64). m-tile mt takes word
//           w = mt%4 of unit vu(g, mt/4): its low half is output row
//           d(mt, g) = 8 vu + 2w, its high half row g+8 = d(mt, g) + 1; prmt
//           pairs two tokens per register.
//        P: the S^T accumulator holds (tokens g, g+8) x (heads 2t, 2t+1); one
//           movmatrix.trans per 8x8 half gives the PV B fragment (tokens 2t..,
//           2t+8..) x (head g) in registers.
//      Swizzle: unit u of row r is stored at slot r*U + (u ^ f(r)), U = D/8,
//      f(r) = 4(r&1) + (r>>1)%4. The row-wise stores, the K reads (rows 2k, 2k+1
//      x a 4-unit block) and the V reads (rows c, c+2, c+4, c+6 x units in the
//      two 4-unit halves) each hit eight distinct 16-byte bank groups per
//      quarter-warp: no bank conflicts.
#pragma once

#include "hga_common.cuh"

namespace hga {

template <int D>
struct TileGeom {
  static constexpr int U = D / 8;          // 16-byte units per row
  static constexpr int RPI = 32 / U;       // rows per coalesced warp load
  static constexpr int NLD = 16 / RPI;     // loads per lane per tensor per tile
  static constexpr int KJ = D / 32;        // K units per row per lane
  static constexpr int VH = D / 64;        // V units per row per lane
  static constexpr int kTileSlots = 16 * U;  // one tensor's 16 rows, uint4 slots
};

__host__ __device__ constexpr int tile_swz(int row, int u) {
  return u ^ (((row & 1) << 2) | ((row >> 1) & 3));
}
__host__ __device__ constexpr int v_unit(int g, int h) { return 8 * h + 4 * (g & 1) + (g >> 1); }

// Output row of O^T held in the low accumulators of m-tile mt by lanes with this g.
__host__ __device__ constexpr int o_row(int mt, int g) { return 8 * v_unit(g, mt >> 2) + 2 * (mt & 3); }

// Q^T (B operand) fragments of all k-steps, shared by the warps of a CTA (they
// attend with the same heads): unit j of lane l is qfrag[j * 32 + l], words
// {x, y} feeding k-step 2j and {z, w} k-step 2j+1.
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

// Coalesced loads of one tensor's tile (rows[0..15], row indices in head_dim
// units; every entry is a readable row) into this lane's registers: x[i] holds
// the lane's unit of rows RPI*i .. RPI*i + RPI-1.
template <int D>
__device__ __forceinline__ void fetch_rows(uint4 (&x)[TileGeom<D>::NLD], const uint32_t* rows,
                                           const uint16_t* base, int lane) {
  using G = TileGeom<D>;
  const int rsub = lane / G::U, u = lane % G::U;
#pragma unroll
  for (int i = 0; i < G::NLD; ++i) x[i] = ldg_stream(base + (int64_t)rows[G::RPI * i + rsub] * D + 8 * u);
}

// Registers -> this warp's swizzled shared tile.
template <int D>
__device__ __forceinline__ void store_rows(uint4* tile, const uint4 (&x)[TileGeom<D>::NLD], int lane) {
  using G = TileGeom<D>;
  const int rsub = lane / G::U, u = lane % G::U;
#pragma unroll
  for (int i = 0; i < G::NLD; ++i) {
    const int row = G::RPI * i + rsub;
    tile[row * G::U + tile_swz(row, u)] = x[i];
  }
}

// S^T of one tile (raw logits): lane (g, t) gets s[0] = (token g, head 2t),
// s[1] = (g, 2t+1), s[2] = (g+8, 2t), s[3] = (g+8, 2t+1). ka[j], kb[j] hold unit
// t + 4j of rows g and g+8 (the K fragment map above).
template <int D>
__device__ __forceinline__ void qk_fragments(float (&s)[4], const uint4 (&ka)[TileGeom<D>::KJ],
                                             const uint4 (&kb)[TileGeom<D>::KJ], const uint4* qfrag, int lane) {
  s[0] = s[1] = s[2] = s[3] = 0.f;
#pragma unroll
  for (int j = 0; j < TileGeom<D>::KJ; ++j) {
    const uint4 qv = qfrag[j * 32 + lane];
    mma_16816(s, ka[j].x, kb[j].x, ka[j].y, kb[j].y, qv.x, qv.y);
    mma_16816(s, ka[j].z, kb[j].z, ka[j].w, kb[j].w, qv.z, qv.w);
  }
}

// Online-softmax update of one tile's logits s (layout of qk_fragments; entries
// at or past n_valid are masked). Returns the PV B fragments (P^T halves, bf16)
// in b0, b1. sl = softmax scale * log2(e).
template <int D>
__device__ __forceinline__ void softmax_update(AttnState<D>& st, float (&s)[4], int n_valid, float sl, int lane,
                                               uint32_t& b0, uint32_t& b1) {
  const int g = lane >> 2;
  if (g >= n_valid) s[0] = s[1] = -INFINITY;
  if (g + 8 >= n_valid) s[2] = s[3] = -INFINITY;
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
  b0 = movmatrix_trans(pack_bf16x2(p0, p1));
  b1 = movmatrix_trans(pack_bf16x2(p2, p3));
}

// QK^T of one tile from the shared K copy, then the online-softmax update.
template <int D>
__device__ __forceinline__ void qk_softmax(AttnState<D>& st, const uint4* ktile, int n_valid,
                                           const uint4* qfrag, float sl, int lane, uint32_t& b0,
                                           uint32_t& b1) {
  using G = TileGeom<D>;
  const int g = lane >> 2;
  const int t = lane & 3;
  uint4 ka[G::KJ], kb[G::KJ];
#pragma unroll
  for (int j = 0; j < G::KJ; ++j) {
    const int u = t + 4 * j;
    ka[j] = ktile[g * G::U + tile_swz(g, u)];
    kb[j] = ktile[(g + 8) * G::U + tile_swz(g + 8, u)];
  }
  float s[4];
  qk_fragments<D>(s, ka, kb, qfrag, lane);
  softmax_update<D>(st, s, n_valid, sl, lane, b0, b1);
}

// O^T += V^T P^T for one tile from the shared V copy.
template <int D>
__device__ __forceinline__ void pv(AttnState<D>& st, const uint4* vtile, uint32_t b0, uint32_t b1,
                                   int lane) {
  using G = TileGeom<D>;
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int h = 0; h < G::VH; ++h) {
    const int u = v_unit(g, h);
    uint4 va[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = 2 * t + (i & 1) + 8 * (i >> 1);
      va[i] = vtile[row * G::U + tile_swz(row, u)];
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t x0 = word_of(va[0], w), x1 = word_of(va[1], w);
      const uint32_t x2 = word_of(va[2], w), x3 = word_of(va[3], w);
      mma_16816(st.o[4 * h + w], prmt(x0, x1, 0x5410), prmt(x0, x1, 0x7632), prmt(x2, x3, 0x5410),
                prmt(x2, x3, 0x7632), b0, b1);
    }
  }
}

// Warp over the tiles tile0, tile0+stride, ... of a staged row table holding
// n_entries real entries (the table is padded to whole tiles with readable
// rows). `tile` is this warp's shared tile (TileGeom<D>::kTileSlots uint4),
// used for K and then for V of each tile; the next tile's K loads are in flight
// during QK^T and softmax, its V loads during PV.
template <int D>
__device__ __forceinline__ void attend_tiles(AttnState<D>& st, const uint32_t* rows, int n_entries,
                                             int tile0, int stride, const uint16_t* K,
                                             const uint16_t* V, const uint4* qfrag, uint4* tile,
                                             float sl, int lane) {
  const int n_tiles = (n_entries + 15) >> 4;
  if (tile0 >= n_tiles) return;
  uint4 kr[TileGeom<D>::NLD], vr[TileGeom<D>::NLD];
  fetch_rows<D>(kr, rows + 16 * tile0, K, lane);
  fetch_rows<D>(vr, rows + 16 * tile0, V, lane);
  for (int tl = tile0; tl < n_tiles; tl += stride) {
    const int nt = tl + stride;
    const bool more = nt < n_tiles;
    store_rows<D>(tile, kr, lane);
    if (more) fetch_rows<D>(kr, rows + 16 * nt, K, lane);
    __syncwarp();
    uint32_t b0, b1;
    qk_softmax<D>(st, tile, n_entries - 16 * tl, qfrag, sl, lane, b0, b1);
    __syncwarp();
    store_rows<D>(tile, vr, lane);
    if (more) fetch_rows<D>(vr, rows + 16 * nt, V, lane);
    __syncwarp();
    pv<D>(st, tile, b0, b1, lane);
    __syncwarp();
  }
}

}  // namespace hga
