// Block-shared two-level routing for chunked prefill.
//
// "Hierarchical Global Attention (HGA)", abstract (chunks, then groups, then
// exact attention); the prefill reading: the queries of one block share a
// routing decision whose chunk score is the maximum, over the block's queries,
// of the head-summed score sum_i q_{p,i} . s_c (and likewise for groups).
//
// One CTA (kRoutedThreads) per (block, KV head). The scores form a small dense
// product [n_q queries x D] . [D x chunks], computed on the tensor cores with
// mma.sync m16n8k16: the fp32 head-summed queries are split into a bf16 high
// part and a bf16 remainder (q = hi + lo, |lo| <= 2^-9 |q|), both multiplied by
// the exact bf16 summaries and accumulated in fp32, which keeps the scores
// within about 2^-16 relative of fp32 arithmetic. The maximum over the queries
// is taken from the accumulator fragments (in-thread, then across the 8 lanes
// that share a column). Top-k uses the same bucket select as decode.
#pragma once

#include "hga_common.cuh"
#include "hga_routed.cuh"

namespace hga {

constexpr int kBlockQ = 64;  // queries per routing block (MMA M = 4 x 16)

struct BlockRouteArgs {
  const uint16_t* q;        // [T][Hq][D]
  int hq, R, T, block;      // block == kBlockQ
  const uint16_t* chunk_sum;  // [Hkv][max_chunks][D] (batch 1, contiguous)
  const uint16_t* group_sum;  // [Hkv][max_chunks][gpc][D]
  int hkv, max_chunks, L;     // L: cache length (routing covers [0, L))
  int growing;                // nonzero: block b routes over [0, L + b * block) (its whole history)
  int C, g, k, G;
  int32_t* idx;    // [n_blocks][Hkv][idx_stride]
  int32_t* n_idx;  // [n_blocks][Hkv]
  int idx_stride;
};

// Shared memory of the block router (the launch adds 8 * n_pad bytes after
// `total` for the bucket-select scratch).
struct BlockRouteSmem {
  int afrag, qs, keys, sel, gmask, hist, misc, gsc, gstart, total;
  __host__ __device__ static int up16(int x) { return (x + 15) & ~15; }
  __host__ __device__ BlockRouteSmem(int D, int n_pad, int kcap, int gk, int gpc) {
    int o = 0;
    afrag = o;  o = up16(o + 4 * 8 * 2 * 32 * 16);  // [m-tile 4][k-step 8][hi/lo 2][lane 32] x uint4 (D = 128)
    qs = o;     o = up16(o + 4 * kBlockQ * D);       // head-summed queries, fp32 [64][D]
    keys = o;   o = up16(o + 8 * n_pad);
    sel = o;    o = up16(o + 4 * kcap);
    gmask = o;  o = up16(o + 4 * kcap);
    hist = o;   o = up16(o + 4 * kHistWords);
    misc = o;   o = up16(o + 4 * 32);
    gsc = o;    o = up16(o + 4 * kcap * gpc);
    gstart = o; o = up16(o + 4 * kcap * gk);
    total = o;
    (void)D;
  }
};

// Column maxima over the 64 queries of scores for 8 summary rows (one N tile).
// The rows are the B operand: lane (g, t) holds units t + 4j of the row of column
// g (load_b_units), matching the permuted head-dim order of the A fragments (see
// hga_attention.cuh). Returns, in lanes with g == 0, the maxima of columns 2t
// and 2t+1. Callers load the next tile's units before scoring the current one.
__device__ __forceinline__ void load_b_units(const uint16_t* my_row, int lane, uint4 (&bu)[4]) {
  const int t = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) bu[j] = ldg_nc(my_row + 8 * (t + 4 * j));
}

// Two row tiles per call: each A fragment read from shared memory feeds both
// tiles' MMAs (the fragments are the scan's shared-memory bandwidth). Every
// (m tile, row tile) accumulator sees the same MMA order as a one-tile scan.
__device__ __forceinline__ void block_scores_tile2(const uint4* afrag, const uint4 (&bu)[2][4], int lane,
                                                   float (&cmax)[2][2]) {
  float acc[2][4][4];
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[u][mt][i] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int j = ks >> 1, p = ks & 1;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
      for (int hl = 0; hl < 2; ++hl) {
        const uint4 a = afrag[((mt * 8 + ks) * 2 + hl) * 32 + lane];
#pragma unroll
        for (int u = 0; u < 2; ++u)
          mma_16816(acc[u][mt], a.x, a.y, a.z, a.w, p ? bu[u][j].z : bu[u][j].x, p ? bu[u][j].w : bu[u][j].y);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      m0 = fmaxf(m0, fmaxf(acc[u][mt][0], acc[u][mt][2]));
      m1 = fmaxf(m1, fmaxf(acc[u][mt][1], acc[u][mt][3]));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, off));
      m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, off));
    }
    cmax[u][0] = m0;
    cmax[u][1] = m1;
  }
}

__global__ void __launch_bounds__(kRoutedThreads) block_route_kernel(const BlockRouteArgs a) {
  constexpr int D = 128;
  extern __shared__ __align__(16) unsigned char br_smem[];
  unsigned char* smem = br_smem;
  const int blk = blockIdx.x / a.hkv, h = blockIdx.x % a.hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int W = kRoutedWarps;
  const int gpc = a.C / a.g, gk = a.G;
  const int L = a.L + (a.growing ? blk * a.block : 0);  // routed history of this block
  const int nf = L / a.C;
  const bool dense = nf <= 2;
  const int n_cand = dense ? 0 : nf - 2;
  const int r = n_cand < a.k ? n_cand : a.k;
  const int n_pad = max(2, a.max_chunks - 2);
  const int kcap = max(1, min(a.k, a.max_chunks - 2));
  const BlockRouteSmem lay(D, n_pad, kcap, gk, gpc);
  uint4* afrag = reinterpret_cast<uint4*>(smem + lay.afrag);
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem + lay.keys);
  int* sel = reinterpret_cast<int*>(smem + lay.sel);
  uint32_t* gmask = reinterpret_cast<uint32_t*>(smem + lay.gmask);
  int* hist = reinterpret_cast<int*>(smem + lay.hist);
  int* misc = reinterpret_cast<int*>(smem + lay.misc);
  float* gsc = reinterpret_cast<float*>(smem + lay.gsc);
  int* gstart = reinterpret_cast<int*>(smem + lay.gstart);

  // Head-summed queries of the block (fp32, 16-byte loads of 8 head dims). Each
  // thread takes two (query, 8-dim unit) items per pass and issues the loads of all
  // their heads before summing (heads in ascending order), 16 loads in flight.
  float* qs = reinterpret_cast<float*>(smem + lay.qs);
  const int q0 = blk * a.block;
  constexpr int kItems = kBlockQ * (D / 8);
  for (int i0 = tid; i0 < kItems; i0 += 2 * kRoutedThreads) {
    uint4 v[2][kMaxHeadsPerKv];
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      const int i = i0 + s2 * kRoutedThreads;
      const int row = i / (D / 8), u = i - row * (D / 8);
      const bool live = i < kItems && q0 + row < a.T;
      const uint16_t* base = a.q + ((int64_t)(q0 + row) * a.hq + (int64_t)h * a.R) * D + 8 * u;
#pragma unroll
      for (int hh = 0; hh < kMaxHeadsPerKv; ++hh)
        v[s2][hh] = (live && hh < a.R) ? ldg_nc(base + (int64_t)hh * D) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      const int i = i0 + s2 * kRoutedThreads;
      const int row = i / (D / 8), u = i - row * (D / 8);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int hh = 0; hh < kMaxHeadsPerKv; ++hh) {
        if (hh < a.R) {
          const uint4 w = v[s2][hh];
          acc[0] += bf16_lo(w.x); acc[1] += bf16_hi(w.x); acc[2] += bf16_lo(w.y); acc[3] += bf16_hi(w.y);
          acc[4] += bf16_lo(w.z); acc[5] += bf16_hi(w.z); acc[6] += bf16_lo(w.w); acc[7] += bf16_hi(w.w);
        }
      }
      if (i < kItems) {
#pragma unroll
        for (int c = 0; c < 8; ++c) qs[row * D + 8 * u + c] = acc[c];
      }
    }
  }
  __syncthreads();
  // A fragments of the head-summed queries, hi/lo bf16 split, permuted head-dim
  // order: fragment (m-tile mt, k-step ks = 2j+p) of lane (g, t): rows 16mt+g and
  // 16mt+g+8, columns 8t + 32j + 4p + {0,1} (a0/a1) and + {2,3} (a2/a3).
  for (int i = tid; i < 4 * 8 * 32; i += kRoutedThreads) {
    const int l = i & 31, ks = (i >> 5) & 7, mt = i >> 8;
    const int g = l >> 2, t = l & 3, j = ks >> 1, p = ks & 1;
    const int col = 8 * t + 32 * j + 4 * p;
    float v[2][4];  // [row g / g+8][col .. col+3]
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
      for (int c = 0; c < 4; ++c) v[rr][c] = qs[(16 * mt + g + 8 * rr) * D + col + c];
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
      for (int c = 0; c < 4; c += 2) {
        const float h0 = __bfloat162float(__float2bfloat16_rn(v[rr][c]));
        const float h1 = __bfloat162float(__float2bfloat16_rn(v[rr][c + 1]));
        // register order: a0 = (row g, cols c0,c1), a1 = (row g+8, c0,c1), a2 = (g, c2,c3), a3 = (g+8, c2,c3)
        const int reg = (c >> 1) * 2 + rr;
        hi[reg] = pack_bf16x2(h0, h1);
        lo[reg] = pack_bf16x2(v[rr][c] - h0, v[rr][c + 1] - h1);
      }
    afrag[((mt * 8 + ks) * 2 + 0) * 32 + l] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    afrag[((mt * 8 + ks) * 2 + 1) * 32 + l] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  for (int i = tid; i < n_pad; i += kRoutedThreads) keys[i] = 0ull;
  __syncthreads();

  const uint16_t* cs = a.chunk_sum + (int64_t)h * a.max_chunks * D;
  const uint16_t* gs = a.group_sum + (int64_t)h * a.max_chunks * gpc * D;
  // chunk scores, 8 candidates per row tile, two row tiles per warp step
  if (n_cand > r) {
    const int n_tiles = (n_cand + 7) / 8;
    const int n_pairs = (n_tiles + 1) / 2;
    // rows past the last candidate repeat it (its scores are not stored)
    auto row_of = [&](int tile) { return cs + (int64_t)(min(tile * 8 + (lane >> 2), n_cand - 1) + 1) * D; };
    uint4 bu[2][4], bn[2][4];
    if (warp < n_pairs) {
      load_b_units(row_of(2 * warp), lane, bu[0]);
      load_b_units(row_of(2 * warp + 1), lane, bu[1]);
    }
    for (int pt = warp; pt < n_pairs; pt += W) {
      if (pt + W < n_pairs) {
        load_b_units(row_of(2 * (pt + W)), lane, bn[0]);
        load_b_units(row_of(2 * (pt + W) + 1), lane, bn[1]);
      }
      float cmax[2][2];
      block_scores_tile2(afrag, bu, lane, cmax);
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int j = 0; j < 4; ++j) bu[u][j] = bn[u][j];
      if ((lane >> 2) == 0) {
        const int t4 = lane & 3;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int ca = (2 * pt + u) * 8 + 2 * t4, cb = ca + 1;
          if (ca < n_cand) keys[ca] = route_key(cmax[u][0], (uint32_t)(ca + 1));
          if (cb < n_cand) keys[cb] = route_key(cmax[u][1], (uint32_t)(cb + 1));
        }
      }
    }
    __syncthreads();
    // scratch for the boundary bucket: n_pad keys right after the layout
    select_top_chunks(keys, n_cand, r, sel, hist, misc, reinterpret_cast<uint64_t*>(smem + lay.total), n_pad);
  } else {
    for (int i = tid; i < r; i += kRoutedThreads) sel[i] = i + 1;
  }
  __syncthreads();

  // group scores: one kept chunk (gpc rows, <= 32) per warp tile of 8 rows
  const bool all_groups = gk >= gpc;
  if (!all_groups) {
    const int tiles_per_chunk = (gpc + 7) / 8;
    auto grow_of = [&](int wt) {
      const int ci = wt / tiles_per_chunk, part = wt - ci * tiles_per_chunk;
      return gs + ((int64_t)sel[ci] * gpc + min(part * 8 + (lane >> 2), gpc - 1)) * D;
    };
    const int n_gt = r * tiles_per_chunk;
    const int n_pairs = (n_gt + 1) / 2;
    // tiles past the last repeat it (their scores are not stored)
    auto grow_at = [&](int wt) { return grow_of(min(wt, n_gt - 1)); };
    uint4 bu[2][4], bn[2][4];
    if (warp < n_pairs) {
      load_b_units(grow_at(2 * warp), lane, bu[0]);
      load_b_units(grow_at(2 * warp + 1), lane, bu[1]);
    }
    for (int pt = warp; pt < n_pairs; pt += W) {
      if (pt + W < n_pairs) {
        load_b_units(grow_at(2 * (pt + W)), lane, bn[0]);
        load_b_units(grow_at(2 * (pt + W) + 1), lane, bn[1]);
      }
      float cmax[2][2];
      block_scores_tile2(afrag, bu, lane, cmax);
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int j = 0; j < 4; ++j) bu[u][j] = bn[u][j];
      if ((lane >> 2) == 0) {
        const int t4 = lane & 3;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int wt = 2 * pt + u;
          if (wt >= n_gt) continue;
          const int ci = wt / tiles_per_chunk, part = wt - ci * tiles_per_chunk;
          const int ja = part * 8 + 2 * t4, jb = ja + 1;
          if (ja < gpc) gsc[ci * gpc + ja] = cmax[u][0];
          if (jb < gpc) gsc[ci * gpc + jb] = cmax[u][1];
        }
      }
    }
    for (int i = tid; i < r; i += kRoutedThreads) gmask[i] = 0u;
    __syncthreads();
    for (int i = tid; i < r * gpc; i += kRoutedThreads) {
      const int ci = i / gpc, j = i - ci * gpc;
      const float tj = gsc[i];
      int rank = 0;
      for (int l = 0; l < gpc; ++l) {
        const float tl = gsc[ci * gpc + l];
        rank += (tl > tj) || (tl == tj && l < j);
      }
      if (rank < gk) atomicOr(&gmask[ci], 1u << j);
    }
    __syncthreads();
  }
  const uint32_t full_mask = gpc >= 32 ? 0xFFFFFFFFu : ((1u << gpc) - 1u);
  for (int i = tid; i < r; i += kRoutedThreads) {
    uint32_t m = all_groups ? full_mask : gmask[i];
    for (int qq = 0; qq < gk; ++qq) {
      const int j = m ? __ffs(m) - 1 : 0;
      m &= m - 1;
      gstart[i * gk + qq] = sel[i] * a.C + j * a.g;
    }
  }
  __syncthreads();
  const int S = dense ? L : a.C + r * gk * a.g + (L - (nf - 1) * a.C);
  const int unit = blk * a.hkv + h;
  const int span = gk * a.g;
  const int Sw = min(S, a.idx_stride);
  if (S > a.idx_stride && tid == 0) report_error(kErrIndex);
  for (int e = tid; e < Sw; e += kRoutedThreads) {
    int tok;
    if (dense || e < a.C) {
      tok = e;
    } else {
      const int u = e - a.C;
      if (u < r * span) {
        const int i = u / span, rem = u - i * span, qq = rem / a.g;
        tok = gstart[i * gk + qq] + (rem - qq * a.g);
      } else {
        tok = (nf - 1) * a.C + (u - r * span);
      }
    }
    a.idx[(int64_t)unit * a.idx_stride + e] = tok;
  }
  if (tid == 0) a.n_idx[unit] = Sw;
}

}  // namespace hga
