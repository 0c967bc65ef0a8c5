// Two-level routing and routed attention for decode, one thread-block cluster
// per (sequence, KV head).
//
// "Hierarchical Global Attention (HGA)", abstract: chunks are picked by their
// summaries first, then the best groups inside them, then attention runs
// exactly over the picked tokens. The first chunk (sink) and the last chunk plus
// any partial tail (local) are always kept, as in the HISA article's two-step
// block filter that always keeps the start and end of the context.
//
// The P CTAs of a cluster split every phase and meet at hardware cluster
// barriers; partial results move through distributed shared memory (DSMEM),
// so nothing goes through global scratch memory:
//   R1  chunk scores: each CTA stages 1/P of the candidate chunk summaries
//       (chunks 1..nf-2) with coalesced cp.async, scores them thread-per-row
//       against the head-summed query (sum_i q_i . s_c = (sum_i q_i) . s_c) and
//       writes the 64-bit keys (score bits, then lower id) into every CTA.
//   --  cluster barrier
//   R2  every CTA finds the k-th largest key of all candidates (bucket select)
//       and keeps the keys at or above it, in ascending chunk order.
//   R3  group scores: each CTA stages and scores the groups of 1/P of the kept
//       chunks and broadcasts a bit mask of the top-G groups per chunk.
//   --  cluster barrier
//   A   attention: the routed list (sink, kept groups, local) is cut into
//       16-token tiles; each CTA takes 1/P of them, its warps take tiles
//       round-robin (hga_attention.cuh).
//   --  cluster barrier, then CTA r combines heads r, r+P, ... from every CTA's
//       (max, denominator, numerator) in DSMEM and writes the output.
//   --  cluster barrier (no CTA leaves while its shared memory is read)
// hga_route runs R1-R3 and writes the list; hga_attend runs A from a given list;
// hga_decode runs everything in one launch.
#pragma once

#include <cooperative_groups.h>

#include "hga_attention.cuh"
#include "hga_common.cuh"

namespace hga {

namespace cg = cooperative_groups;

enum RoutedMode : int { kModeRoute = 1, kModeAttend = 2, kModeDecode = 3 };

constexpr int kRoutedWarps = 6;
constexpr int kRoutedThreads = kRoutedWarps * 32;
constexpr int kBuckets = 1024;             // bucket-select histogram size
// Histograms are stored with one padding word after every 32 buckets
// (hist_index), so that warp lanes reading buckets a multiple of 32 apart hit
// distinct shared-memory banks; kHistWords words hold kBuckets buckets.
constexpr int kHistWords = kBuckets + kBuckets / 32;
__host__ __device__ constexpr int hist_index(int b) { return b + (b >> 5); }
// misc[] (32 ints): [0..5] select state, [8..15] per-warp min, [16..23] per-warp
// max, [24..31] per-warp scan totals
static_assert(kRoutedWarps <= 8, "misc[] holds at most 8 per-warp slots");
constexpr int kStageBytes = 32 * 1024;     // routing: double-buffered summary staging
// Cluster combine: CTA n % P finalises head n and receives P * ceil(R / P)
// partials, at most 16 for R <= 8 and P <= 16.
constexpr int kGatherSlots = 16;

struct RoutedArgs {
  KvView kv;
  SumView sv;
  const uint16_t* q;  // [B][Hq][D]
  int hq, R;
  int C, g, k, G;     // routing parameters (G already <= C/g)
  int n_pad;          // >= max candidates (max_chunks - 2), >= 2
  int kcap;           // >= kept chunks for any length (min(k, max_chunks - 2)), >= 1
  int k_tok;          // block-then-token routing: tokens kept by the token step
  float scale_log2;   // softmax scale * log2(e)
  float* out;         // [B][Hq][D]
  float* lse;         // [B][Hq] or null
  int32_t* idx_out;   // [B][Hkv][idx_stride] or null
  int32_t* n_idx_out; // [B][Hkv] or null
  const int32_t* idx_in;
  const int32_t* n_idx_in;
  int idx_stride;
  float* logits;      // block-then-token decode: per-head logits of the token step's candidates,
                      // [B * Hkv][lg_stride / 8][8] (null: the attention recomputes them from K)
  int64_t lg_stride;  // floats per (sequence, KV head)
};

// Shared-memory carve-up (byte offsets), identical on host and device. One
// union region serves, in turn, the routing keys plus the summary staging
// area, the per-warp attention tiles, and the per-warp partial outputs.
struct RoutedSmem {
  int qsum, sel, gmask, gstart, rows, red_m, red_l, cta_o, cta_m, cta_l, qfrag, hist, misc, gsc,
      uni, keys, stage, stage_rows, tiles, red_o, total;
  __host__ __device__ static int up16(int x) { return (x + 15) & ~15; }
  __host__ __device__ RoutedSmem(int D, int n_pad, int kcap, int gk, int gpc) {
    int o = 0;
    qsum = o;    o = up16(o + 4 * D);
    sel = o;     o = up16(o + 4 * kcap);
    gmask = o;   o = up16(o + 4 * kcap);
    gstart = o;  o = up16(o + 4 * kcap * gk);
    rows = o;    o = up16(o + 4 * kEntryBatch);
    red_m = o;   o = up16(o + 4 * kRoutedWarps * kMaxHeadsPerKv);
    red_l = o;   o = up16(o + 4 * kRoutedWarps * kMaxHeadsPerKv);
    cta_o = o;   o = up16(o + 4 * kGatherSlots * D);
    cta_m = o;   o = up16(o + 4 * kGatherSlots);
    cta_l = o;   o = up16(o + 4 * kGatherSlots);
    qfrag = o;   o = up16(o + 16 * 32 * (D / 32));
    hist = o;    o = up16(o + 4 * kHistWords);
    misc = o;    o = up16(o + 4 * 32);
    // union: {keys, staging} during routing | per-warp tiles | partial outputs
    uni = o;
    keys = o;
    stage = up16(keys + 8 * n_pad);
    stage_rows = kStageBytes / (2 * D);
    tiles = o;
    red_o = o;
    int u = stage + kStageBytes - o;
    const int tiles_bytes = kRoutedWarps * 16 * D * 2;
    const int red_bytes = 4 * kRoutedWarps * kMaxHeadsPerKv * D;
    if (tiles_bytes > u) u = tiles_bytes;
    if (red_bytes > u) u = red_bytes;
    o = up16(o + u);
    gsc = o;     o = up16(o + 4 * kcap * gpc);
    total = o;
  }
};

// Block-wide exclusive prefix sum of one int per thread (kRoutedThreads).
__device__ __forceinline__ int block_exclusive_scan(int x, int* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += wsum[w];
  __syncthreads();
  return before + incl - x;
}

// Staged summary rows: unit u of staged row i sits at slot i*U + (u ^ (i % U)),
// so row-wise stores and thread-per-row reads are both bank-conflict-free.
template <int D>
__device__ __forceinline__ int stage_slot(int i, int u) {
  return i * (D / 8) + (u ^ (i & (D / 8 - 1)));
}

// Head-summed score of staged row i: qsum . row (fp32).
template <int D>
__device__ __forceinline__ float staged_row_dot(const uint4* stage, int i, const float* qsum) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int u = 0; u < D / 8; ++u) {
    const uint4 v = stage[stage_slot<D>(i, u)];
    const float4 a = *reinterpret_cast<const float4*>(qsum + 8 * u);
    const float4 c = *reinterpret_cast<const float4*>(qsum + 8 * u + 4);
    s0 = fmaf(bf16_lo(v.x), a.x, s0);
    s1 = fmaf(bf16_hi(v.x), a.y, s1);
    s0 = fmaf(bf16_lo(v.y), a.z, s0);
    s1 = fmaf(bf16_hi(v.y), a.w, s1);
    s0 = fmaf(bf16_lo(v.z), c.x, s0);
    s1 = fmaf(bf16_hi(v.z), c.y, s1);
    s0 = fmaf(bf16_lo(v.w), c.z, s0);
    s1 = fmaf(bf16_hi(v.w), c.w, s1);
  }
  return s0 + s1;
}

// Stream n_rows summary rows through the staging area in two alternating
// buffers (cp.async groups), so the copies of block i+1 are in flight while
// block i is scored. src(row) gives the global address of a row; consume(buf,
// first_row, n) scores rows first_row .. first_row+n-1 staged at buf
// (stage_slot layout, local row index). Every thread of the CTA must call it.
template <int D, typename Src, typename Consume>
__device__ __forceinline__ void stream_rows(uint4* stage, int stage_rows, int n_rows, Src src,
                                            Consume consume) {
  constexpr int U = D / 8;
  const int half = stage_rows / 2;
  auto issue = [&](int first, uint4* buf) {
    const int n = min(half, n_rows - first);
    for (int p = threadIdx.x; p < n * U; p += kRoutedThreads) {
      const int i = p / U, u = p - i * U;
      cp_async16(buf + stage_slot<D>(i, u), src(first + i) + 8 * u);
    }
  };
  uint4* bufs[2] = {stage, stage + half * U};
  if (0 < n_rows) issue(0, bufs[0]);
  cp_async_commit();
  if (half < n_rows) issue(half, bufs[1]);
  cp_async_commit();
  int which = 0;
  for (int first = 0; first < n_rows; first += half) {
    cp_async_wait<1>();
    __syncthreads();
    consume(bufs[which], first, min(half, n_rows - first));
    __syncthreads();
    if (first + 2 * half < n_rows) issue(first + 2 * half, bufs[which]);
    cp_async_commit();
    which ^= 1;
  }
  cp_async_wait<0>();
}

// Warp 0 finds the bucket holding the need-th largest key (1 <= need <= keys
// counted): misc[0] = that bucket, misc[1] = keys in the buckets above it. Lane l
// sums the NB/32 buckets NB-1-(NB/32)l-k (k ascending = buckets descending), a
// warp scan finds the lane whose range holds the need-th key, then one bucket
// of that range per lane and a second scan find the bucket. The padded layout
// makes both reads free of bank conflicts.
template <int NB>
__device__ __forceinline__ void find_boundary_bucket(const int* hist, int need, int* misc) {
  static_assert(NB % 32 == 0 && NB / 32 <= 32, "one bucket range per lane, at most 32 buckets each");
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x & 31;
  constexpr int PER = NB / 32;
  int tot = 0;
#pragma unroll
  for (int k = 0; k < PER; ++k) tot += hist[hist_index(NB - 1 - PER * lane - k)];
  int incl = tot;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  const int excl = incl - tot;
  const uint32_t hit = __ballot_sync(0xFFFFFFFFu, excl < need && need <= incl);
  const int L = __ffs(hit) - 1;
  const int above = __shfl_sync(0xFFFFFFFFu, excl, L);
  const int bk = NB - 1 - PER * L - lane;  // this lane's bucket of range L
  const int v = lane < PER ? hist[hist_index(bk)] : 0;
  int pre = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, pre, off);
    if (lane >= off) pre += t;
  }
  const uint32_t hit2 = __ballot_sync(0xFFFFFFFFu, lane < PER && above + pre >= need);
  if (lane == __ffs(hit2) - 1) {
    misc[0] = bk;
    misc[1] = above + pre - v;
  }
}

// Top-r selection over n unique keys; keys[i] belongs to candidate chunk i+1
// (key = order-preserving score bits << 32 | ~id, so larger key = higher score,
// then lower id: the oracle's order). Finds the r-th largest key K_r exactly and
// writes the ids of all keys >= K_r, ascending, to sel[0..r):
//   1. bucket the 32-bit score parts linearly between their block min and max
//      (a monotone map), histogram, and find the bucket b* holding the r-th;
//   2. compact the keys of b* and rank them exactly (64-bit compare) to get K_r;
//   3. ordered compaction of keys >= K_r (candidate order = ascending ids).
// scratch must hold scratch_cap keys; if b* holds more, ranking falls back to
// scanning all n keys (correct, slower; only for near-constant scores).
template <int NB = kBuckets>
__device__ __forceinline__ void select_top_chunks(const uint64_t* keys, int n, int r, int* sel,
                                                  int* hist, int* misc, uint64_t* scratch,
                                                  int scratch_cap) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int i = tid; i < n; i += kRoutedThreads) {
    const uint32_t u = (uint32_t)(keys[i] >> 32);
    lo = min(lo, u);
    hi = max(hi, u);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, off));
    hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, off));
  }
  if (lane == 0) {
    misc[8 + warp] = (int)lo;
    misc[16 + warp] = (int)hi;
  }
  for (int i = tid; i < hist_index(NB); i += kRoutedThreads) hist[i] = 0;
  if (tid == 0) misc[2] = 0;
  __syncthreads();
  lo = 0xFFFFFFFFu;
  hi = 0u;
#pragma unroll
  for (int w = 0; w < kRoutedWarps; ++w) {
    lo = min(lo, (uint32_t)misc[8 + w]);
    hi = max(hi, (uint32_t)misc[16 + w]);
  }
  const float scale = (float)NB / ((float)(hi - lo) + 1.0f);
  auto bucket = [&](uint32_t u) { return min(NB - 1, (int)((float)(u - lo) * scale)); };
  for (int i = tid; i < n; i += kRoutedThreads) atomicAdd(&hist[hist_index(bucket((uint32_t)(keys[i] >> 32)))], 1);
  __syncthreads();
  find_boundary_bucket<NB>(hist, r, misc);
  __syncthreads();
  const int bstar = misc[0], need = r - misc[1];
  const int members = hist[hist_index(bstar)];
  const bool in_scratch = members <= scratch_cap;
  if (in_scratch) {
    for (int i = tid; i < n; i += kRoutedThreads) {
      const uint64_t key = keys[i];
      if (bucket((uint32_t)(key >> 32)) == bstar) scratch[atomicAdd(&misc[2], 1)] = key;
    }
    __syncthreads();
    for (int m = tid; m < members; m += kRoutedThreads) {
      const uint64_t km = scratch[m];
      int rank = 0;
      for (int j = 0; j < members; ++j) rank += scratch[j] > km;
      if (rank == need - 1) {
        misc[4] = (int)(uint32_t)(km >> 32);
        misc[5] = (int)(uint32_t)(km & 0xFFFFFFFFu);
      }
    }
  } else {
    for (int i = tid; i < n; i += kRoutedThreads) {
      const uint64_t km = keys[i];
      if (bucket((uint32_t)(km >> 32)) != bstar) continue;
      int rank = 0;
      for (int j = 0; j < n; ++j) {
        const uint64_t kj = keys[j];
        rank += (kj > km) && bucket((uint32_t)(kj >> 32)) == bstar;
      }
      if (rank == need - 1) {
        misc[4] = (int)(uint32_t)(km >> 32);
        misc[5] = (int)(uint32_t)(km & 0xFFFFFFFFu);
      }
    }
  }
  __syncthreads();
  const uint64_t kth = ((uint64_t)(uint32_t)misc[4] << 32) | (uint64_t)(uint32_t)misc[5];
  const int per = (n + kRoutedThreads - 1) / kRoutedThreads;
  const int s0 = min(n, tid * per), s1 = min(n, s0 + per);
  int cnt = 0;
  for (int i = s0; i < s1; ++i) cnt += keys[i] >= kth;
  int pos = block_exclusive_scan(cnt, misc + 24);
  for (int i = s0; i < s1; ++i)
    if (keys[i] >= kth && pos < r) sel[pos++] = (int)route_key_id(keys[i]);
}

// Per-warp softmax states -> CTA partial (shared memory) -> output. A single-CTA
// cluster writes out/lse directly; otherwise the CTAs combine their partials
// through DSMEM, CTA cr finalising heads cr, cr + P, ... Every thread of every
// CTA of the cluster must call it.
template <int D>
__device__ __forceinline__ void finish_attention(AttnState<D>& st, const RoutedArgs& a, cg::cluster_group& cluster,
                                                 int P, int cr, int b, int h, float* red_o, float* red_m,
                                                 float* red_l, float* cta_o, float* cta_m, float* cta_l) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __syncthreads();  // every warp is done with its tile before red_o reuses the region

  // warp partials -> shared memory
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    st.l0 += __shfl_xor_sync(0xFFFFFFFFu, st.l0, off);
    st.l1 += __shfl_xor_sync(0xFFFFFFFFu, st.l1, off);
  }
  {
    const int g8 = lane >> 2, t4 = lane & 3;
    const int h0 = 2 * t4, h1 = 2 * t4 + 1;
    float* wo = red_o + warp * kMaxHeadsPerKv * D;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      const int d0 = o_row(mt, g8);
      wo[h0 * D + d0] = st.o[mt][0];
      wo[h1 * D + d0] = st.o[mt][1];
      wo[h0 * D + d0 + 1] = st.o[mt][2];
      wo[h1 * D + d0 + 1] = st.o[mt][3];
    }
    if (g8 == 0) {
      red_m[warp * kMaxHeadsPerKv + h0] = st.m0;
      red_m[warp * kMaxHeadsPerKv + h1] = st.m1;
      red_l[warp * kMaxHeadsPerKv + h0] = st.l0;
      red_l[warp * kMaxHeadsPerKv + h1] = st.l1;
    }
  }
  __syncthreads();
  // CTA combine over warps. A single-CTA cluster writes the output directly;
  // otherwise head n is finalised by CTA n % P, and every CTA pushes its
  // partial of head n into that CTA's gather slot cr * HPC + n / P (remote
  // stores, then one cluster barrier; the finalising reads are local).
  const int HPC = (a.R + P - 1) / P;
  for (int i = tid; i < a.R * D; i += kRoutedThreads) {
    const int n = i / D, dd = i - n * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kRoutedWarps; ++w) M = fmaxf(M, red_m[w * kMaxHeadsPerKv + n]);
    float acc = 0.f, den = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kRoutedWarps; ++w) {
        const float f = ex2(red_m[w * kMaxHeadsPerKv + n] - M);  // -inf -> 0
        acc = fmaf(red_o[(w * kMaxHeadsPerKv + n) * D + dd], f, acc);
        den = fmaf(red_l[w * kMaxHeadsPerKv + n], f, den);
      }
    }
    if (P == 1) {
      const int64_t head = (int64_t)b * a.hq + (int64_t)h * a.R + n;
      a.out[head * D + dd] = den > 0.f ? acc / den : 0.f;
      if (dd == 0 && a.lse != nullptr)
        a.lse[head] = den > 0.f ? (M + __log2f(den)) * 0.69314718055994530942f : -INFINITY;
    } else {
      const int owner = n % P, slot = cr * HPC + n / P;
      cluster.map_shared_rank(cta_o, owner)[slot * D + dd] = acc;
      if (dd == 0) {
        cluster.map_shared_rank(cta_m, owner)[slot] = M;
        cluster.map_shared_rank(cta_l, owner)[slot] = den;
      }
    }
  }
  if (P > 1) {
    // After this barrier no CTA touches another's shared memory, so there is
    // no closing barrier.
    cluster.sync();
    const int my_heads = cr < a.R ? (a.R - cr + P - 1) / P : 0;
    for (int i = tid; i < my_heads * D; i += kRoutedThreads) {
      const int jj = i / D, dd = i - jj * D, n = cr + P * jj;
      float M = -INFINITY;
      for (int pr = 0; pr < P; ++pr) M = fmaxf(M, cta_m[pr * HPC + jj]);
      float acc = 0.f, den = 0.f;
      if (M != -INFINITY) {
        for (int pr = 0; pr < P; ++pr) {
          const float f = ex2(cta_m[pr * HPC + jj] - M);  // -inf -> 0
          acc = fmaf(cta_o[(pr * HPC + jj) * D + dd], f, acc);
          den = fmaf(cta_l[pr * HPC + jj], f, den);
        }
      }
      const int64_t head = (int64_t)b * a.hq + (int64_t)h * a.R + n;
      a.out[head * D + dd] = den > 0.f ? acc / den : 0.f;
      if (dd == 0 && a.lse != nullptr)
        a.lse[head] = den > 0.f ? (M + __log2f(den)) * 0.69314718055994530942f : -INFINITY;
    }
  }
}

template <int D, int MODE>
__global__ void __launch_bounds__(kRoutedThreads, 2) routed_kernel(const RoutedArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ uint32_t fallback_row;
  cg::cluster_group cluster = cg::this_cluster();
  const int P = (int)cluster.num_blocks();
  const int cr = (int)cluster.block_rank();
  const int unit = blockIdx.x / P;
  const int hkv = a.kv.hkv;
  const int b = unit / hkv, h = unit % hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr bool kRouting = (MODE & kModeRoute) != 0;
  constexpr bool kAttention = (MODE & kModeAttend) != 0;

  const int gk = a.G;
  const RoutedSmem lay(D, a.n_pad, a.kcap, gk, a.C / a.g);
  float* qsum = reinterpret_cast<float*>(smem + lay.qsum);
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem + lay.keys);
  uint4* stage = reinterpret_cast<uint4*>(smem + lay.stage);
  const int stage_rows = lay.stage_rows;
  int* hist = reinterpret_cast<int*>(smem + lay.hist);
  int* misc = reinterpret_cast<int*>(smem + lay.misc);
  float* gsc = reinterpret_cast<float*>(smem + lay.gsc);
  int* sel = reinterpret_cast<int*>(smem + lay.sel);
  uint32_t* gmask = reinterpret_cast<uint32_t*>(smem + lay.gmask);
  int* gstart = reinterpret_cast<int*>(smem + lay.gstart);
  uint32_t* rows = reinterpret_cast<uint32_t*>(smem + lay.rows);
  float* red_o = reinterpret_cast<float*>(smem + lay.red_o);
  float* red_m = reinterpret_cast<float*>(smem + lay.red_m);
  float* red_l = reinterpret_cast<float*>(smem + lay.red_l);
  float* cta_o = reinterpret_cast<float*>(smem + lay.cta_o);
  float* cta_m = reinterpret_cast<float*>(smem + lay.cta_m);
  float* cta_l = reinterpret_cast<float*>(smem + lay.cta_l);
  uint4* qfrag = reinterpret_cast<uint4*>(smem + lay.qfrag);
  uint4* tile = reinterpret_cast<uint4*>(smem + lay.tiles) + warp * TileGeom<D>::kTileSlots;

  const bool paged = a.kv.page_table != nullptr;
  const int L = a.kv.length(b);
  const int C = a.C, g = a.g, gpc = C / g;
  const uint16_t* qb = a.q + ((int64_t)b * a.hq + (int64_t)h * a.R) * D;

  // ------------------------------------------------------------- routing
  const int nf = L / C;
  const bool dense = nf <= 2;
  const int n_cand = dense ? 0 : nf - 2;
  const int r = n_cand < a.k ? n_cand : a.k;
  int S = 0;  // routed entries

  // physical page of chunk c (paged caches; 0 after reporting a bad entry)
  auto chunk_page = [&](int c) -> int {
    if (!paged) return 0;
    const int page = __ldg(a.kv.page_table + (int64_t)b * a.kv.max_pages + c);
    if ((unsigned)page >= (unsigned)a.kv.num_pages) {
      report_error(kErrPage);
      return 0;  // read a real row; results after a reported error are unspecified
    }
    return page;
  };

  if (kRouting) {
    // Peers write into this CTA's shared memory in R1; every CTA of the cluster
    // must have started first. Arrive now, wait just before the first remote store.
    cluster_arrive_relaxed();
    for (int e = tid; e < D; e += kRoutedThreads) {
      float s = 0.f;
      for (int i = 0; i < a.R; ++i) s += bf16_to_f(qb[(int64_t)i * D + e]);
      qsum[e] = s;
    }
    __syncthreads();
    cluster_wait();

    // R1: score this CTA's share of the candidates; broadcast keys to the cluster.
    const bool select_needed = n_cand > r;
    if (select_needed) {
      const int c0 = (int)((int64_t)n_cand * cr / P), c1 = (int)((int64_t)n_cand * (cr + 1) / P);
      stream_rows<D>(
          stage, stage_rows, c1 - c0,
          [&](int i) {
            const int c = c0 + i + 1;
            return a.sv.chunk + a.sv.chunk_off(paged, b, h, hkv, c, chunk_page(c));
          },
          [&](const uint4* buf, int first, int n) {
            for (int i = tid; i < n; i += kRoutedThreads) {
              const int cand = c0 + first + i;
              const uint64_t key = route_key(staged_row_dot<D>(buf, i, qsum), (uint32_t)(cand + 1));
              for (int pr = 0; pr < P; ++pr) cluster.map_shared_rank(keys, pr)[cand] = key;
            }
          });
    }
    cluster.sync();

    // R2: top-r chunks, ascending ids (every CTA, from the full key set).
    if (select_needed) {
      select_top_chunks(keys, n_cand, r, sel, hist, misc, reinterpret_cast<uint64_t*>(stage),
                        (stage_rows * 2 * D) / 8);
    } else {
      for (int i = tid; i < r; i += kRoutedThreads) sel[i] = i + 1;
    }
    __syncthreads();

    // R3: group top-G inside this CTA's share of the kept chunks.
    const bool all_groups = gk >= gpc;
    if (!all_groups) {
      const int s0 = (int)((int64_t)r * cr / P), s1 = (int)((int64_t)r * (cr + 1) / P);
      const int n_rows = (s1 - s0) * gpc;
      for (int i = tid; i < s1 - s0; i += kRoutedThreads) gmask[s0 + i] = 0u;
      stream_rows<D>(
          stage, stage_rows, n_rows,
          [&](int i) {
            const int ci = i / gpc, j = i - ci * gpc;
            const int c = sel[s0 + ci];
            return a.sv.group + a.sv.group_off(paged, b, h, hkv, c, chunk_page(c)) + (int64_t)j * D;
          },
          [&](const uint4* buf, int first, int n) {
            for (int i = tid; i < n; i += kRoutedThreads) gsc[first + i] = staged_row_dot<D>(buf, i, qsum);
          });
      __syncthreads();
      for (int i = tid; i < n_rows; i += kRoutedThreads) {
        const int ci = i / gpc, j = i - ci * gpc;
        const float tj = gsc[i];
        const float* row_scores = gsc + ci * gpc;
        int rank = 0;
        for (int l = 0; l < gpc; ++l) {
          const float tl = row_scores[l];
          rank += (tl > tj) || (tl == tj && l < j);
        }
        if (rank < gk) atomicOr(&gmask[s0 + ci], 1u << j);
      }
      __syncthreads();
      for (int ci = tid; ci < s1 - s0; ci += kRoutedThreads) {
        const uint32_t m = gmask[s0 + ci];
        for (int pr = 0; pr < P; ++pr)
          if (pr != cr) cluster.map_shared_rank(gmask, pr)[s0 + ci] = m;
      }
    }
    cluster.sync();

    // Group starts of the routed list, per kept chunk in ascending group order.
    const uint32_t full_mask = gpc >= 32 ? 0xFFFFFFFFu : ((1u << gpc) - 1u);
    for (int i = tid; i < r; i += kRoutedThreads) {
      uint32_t m = all_groups ? full_mask : gmask[i];
      for (int qq = 0; qq < gk; ++qq) {
        const int j = m ? __ffs(m) - 1 : 0;
        m &= m - 1;
        gstart[i * gk + qq] = sel[i] * C + j * g;
      }
    }
    __syncthreads();
    S = dense ? L : C + r * gk * g + (L - (nf - 1) * C);
  } else {
    S = __ldg(a.n_idx_in + unit);
    if (S < 0 || S > a.idx_stride) {
      if (tid == 0 && cr == 0) report_error(kErrIndex);
      S = 0;
    }
  }

  // routed entry -> token position
  const int span = gk * g;
  auto entry_token = [&](int e) -> int {
    if (!kRouting) return __ldg(a.idx_in + (int64_t)unit * a.idx_stride + e);
    if (dense || e < C) return e;
    const int u = e - C;
    if (u < r * span) {
      const int i = u / span, rem = u - i * span;
      const int qq = rem / g;
      return gstart[i * gk + qq] + (rem - qq * g);
    }
    return (nf - 1) * C + (u - r * span);
  };

  if (kRouting && a.idx_out != nullptr) {
    int Sw = S;
    if (Sw > a.idx_stride) {
      if (tid == 0 && cr == 0) report_error(kErrIndex);
      Sw = a.idx_stride;
    }
    const int e0 = (int)((int64_t)Sw * cr / P), e1 = (int)((int64_t)Sw * (cr + 1) / P);
    for (int e = e0 + tid; e < e1; e += kRoutedThreads)
      a.idx_out[(int64_t)unit * a.idx_stride + e] = entry_token(e);
    if (cr == 0 && tid == 0) a.n_idx_out[unit] = S;
  }

  if (kAttention) {
    // ------------------------------------------------------------ attention
    AttnState<D> st;
    st.init();
    stage_q_fragments<D>(qfrag, qb, a.R, tid, kRoutedThreads);
    const int n_tiles = (S + 15) / 16;
    const int t0 = (int)((int64_t)n_tiles * cr / P), t1 = (int)((int64_t)n_tiles * (cr + 1) / P);
    const int e_begin = 16 * t0, e_end = min(16 * t1, S);
    const uint16_t* Kp = a.kv.k;
    const uint16_t* Vp = a.kv.v;
    for (int eb = e_begin; eb < e_end; eb += kEntryBatch) {
      const int n_e = min(kEntryBatch, e_end - eb);
      const int n_t = (n_e + 15) / 16;
      __syncthreads();
      for (int i = tid; i < n_t * 16; i += kRoutedThreads) {
        uint32_t row = kInvalidRow;
        if (i < n_e) {
          const int tok = entry_token(eb + i);
          if (tok >= 0 && tok < L) {
            row = a.kv.row(b, h, tok);
          } else {
            report_error(kErrIndex);
          }
        }
        rows[i] = row;
      }
      __syncthreads();
      // Entries without a readable row (padding past n_e, or a bad token / page
      // that was just reported) read the batch's first readable row instead and
      // are masked (padding) or contribute unspecified values (reported errors).
      if (tid < 32) {
        uint32_t first = kInvalidRow;
        for (int i0 = 0; i0 < n_e && first == kInvalidRow; i0 += 32) {
          const uint32_t v = (i0 + lane < n_e) ? rows[i0 + lane] : kInvalidRow;
          const uint32_t ok = __ballot_sync(0xFFFFFFFFu, v != kInvalidRow);
          if (ok) first = __shfl_sync(0xFFFFFFFFu, v, __ffs(ok) - 1);
        }
        if (lane == 0) fallback_row = first == kInvalidRow ? 0u : first;
      }
      __syncthreads();
      for (int i = tid; i < n_t * 16; i += kRoutedThreads)
        if (rows[i] == kInvalidRow) rows[i] = fallback_row;
      __syncthreads();
      attend_tiles<D>(st, rows, n_e, warp, kRoutedWarps, Kp, Vp, qfrag, tile, a.scale_log2, lane);
    }
    finish_attention<D>(st, a, cluster, P, cr, b, h, red_o, red_m, red_l, cta_o, cta_m, cta_l);
  }
}

}  // namespace hga
