// Block-then-token routed decode: a coarse filter on block summaries, then a
// token-level indexer inside the kept blocks, then exact attention over the
// kept tokens; one thread-block cluster of P CTAs per (sequence, KV head).
//
// "Hierarchical Indexing Sparse Attention" (HISA article, shijienb.com
// summary): the text is cut into fixed-size blocks with one feature vector
// each; the blocks are scored with the indexer's own rule and the best ones
// kept, always with the beginning and the end of the text; only the tokens of
// the kept blocks are then scored token by token, which brings the indexer's
// O(L^2) cost down to O(L^2/B + L m B). Here the blocks are the chunks with
// their mean-of-keys summaries, and the scoring rule of both steps is the
// head-summed one of the two-level route (sum over the query heads of a KV
// head of q_i . v, no softmax scale).
// Phases:
//   R1  chunk scores of candidates 1..nf-2 (as in decode_kernel: 16-row
//       register batches, halving-butterfly reduction, keys to every CTA)
//   --  cluster barrier
//   R2  top-m chunks (select_top_chunks, 256 buckets, ascending ids), in
//       every CTA
//   T1  the candidate tokens, [0, C) + the kept chunks' tokens + [(nf-1)C, L)
//       (every token when nf <= 2), are split over the CTAs in batches of 16
//       consecutive positions and scored the same way from registers; their
//       64-bit keys (score bits, then lower candidate index, which orders like
//       the position) and the score range go to every CTA. With a logits
//       workspace (hga_decode_hisa_ws) a batch is instead one QK^T MMA tile
//       (tokens x query heads, K fragments loaded straight from HBM): the score
//       is the sum of the tile's per-head logits, and the logits are stored
//       (32 B per candidate) for phase A
//   --  cluster barrier (skipped, with T1 and T2, when the candidates are no
//       more than the tokens to keep)
//   T2  top k_tok tokens (select_top_keys on the score range T1 publishes,
//       ascending positions), in every CTA
//   A   exact attention over the kept tokens: 16-token tiles split over the
//       CTAs and round-robin over the warps (hga_attention.cuh), rows staged
//       in batches of kEntryBatch entries; with the logits workspace the tiles
//       load the stored logits and gather only V (the kept tokens' K is not
//       read a second time)
//   --  warp -> CTA -> cluster softmax combine (finish_attention)
#pragma once

#include "hga_decode.cuh"

namespace hga {

// score-range table in HisaSmem::tmm (floats): token-score range per CTA of
// the cluster, then per-warp scratch
constexpr int kTmmTok = 0, kTmmWarp = 2 * kGatherSlots;
// chunk select: the bit-pattern bucket select of the two-level route with a
// smaller histogram (measured faster here than 1024 buckets or select_top_keys)
constexpr int kChunkBuckets = 256;

// Shared-memory carve-up (byte offsets), identical on host and device. The
// union region holds the chunk keys, the token keys and the select scratch,
// then the per-warp attention tiles, then the per-warp partial outputs.
struct HisaSmem {
  int qsum, sel, pages, red_m, red_l, cta_o, cta_m, cta_l, qfrag, hist, misc, kred, tmm, rows, tsel, uni, ckeys,
      tkeys, scratch, tiles, red_o, total;
  __host__ __device__ static int up16(int x) { return (x + 15) & ~15; }
  // n_tok_pad >= the most candidate tokens at any length, k_tok = tokens kept
  __host__ __device__ HisaSmem(int D, int n_pad, int kcap, int n_tok_pad, int k_tok) {
    int o = 0;
    qsum = o;    o = up16(o + 4 * D);
    sel = o;     o = up16(o + 4 * kcap);
    pages = o;   o = up16(o + 4 * (n_pad + 4));
    red_m = o;   o = up16(o + 4 * kRoutedWarps * kMaxHeadsPerKv);
    red_l = o;   o = up16(o + 4 * kRoutedWarps * kMaxHeadsPerKv);
    cta_o = o;   o = up16(o + 4 * kGatherSlots * D);
    cta_m = o;   o = up16(o + 4 * kGatherSlots);
    cta_l = o;   o = up16(o + 4 * kGatherSlots);
    qfrag = o;   o = up16(o + 16 * 32 * (D / 32));
    hist = o;    o = up16(o + 4 * kHistWords);
    misc = o;    o = up16(o + 4 * 32);
    kred = o;    o = up16(o + 8 * (2 * kRoutedWarps + 2));
    tmm = o;     o = up16(o + 4 * (kTmmWarp + 2 * kRoutedWarps));
    rows = o;    o = up16(o + 4 * kEntryBatch);
    tsel = o;    o = up16(o + 4 * k_tok);
    uni = o;
    ckeys = o;
    tkeys = up16(ckeys + 8 * n_pad);
    scratch = up16(tkeys + 8 * n_tok_pad);
    tiles = o;
    red_o = o;
    int u = scratch + 8 * kDecodeScratchKeys - o;
    const int tiles_bytes = kRoutedWarps * 16 * D * 2;
    const int red_bytes = 4 * kRoutedWarps * kMaxHeadsPerKv * D;
    if (tiles_bytes > u) u = tiles_bytes;
    if (red_bytes > u) u = red_bytes;
    o = up16(o + u);
    total = o;
  }
};

// Least lo and greatest hi over the CTA's threads, written to slot cr of the
// table `tab` of every CTA of the cluster (tab[2 cr], tab[2 cr + 1]); the
// caller's next cluster barrier publishes them. Every thread of the CTA calls it.
__device__ __forceinline__ void publish_range(float lo, float hi, float* tmm, int tab, cg::cluster_group& cluster,
                                              int P, int cr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, off));
  }
  if (lane == 0) {
    tmm[kTmmWarp + 2 * warp] = lo;
    tmm[kTmmWarp + 2 * warp + 1] = hi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 1; w < kRoutedWarps; ++w) {
      lo = fminf(lo, tmm[kTmmWarp + 2 * w]);
      hi = fmaxf(hi, tmm[kTmmWarp + 2 * w + 1]);
    }
    for (int pr = 0; pr < P; ++pr) {
      float* dst = cluster.map_shared_rank(tmm, pr) + tab;
      dst[2 * cr] = lo;
      dst[2 * cr + 1] = hi;
    }
  }
}

// The range over the P slots of table `tab` (after the cluster barrier).
__device__ __forceinline__ void cluster_range(const float* tmm, int tab, int P, float& lo, float& hi) {
  lo = tmm[tab];
  hi = tmm[tab + 1];
  for (int pr = 1; pr < P; ++pr) {
    lo = fminf(lo, tmm[tab + 2 * pr]);
    hi = fmaxf(hi, tmm[tab + 2 * pr + 1]);
  }
}

constexpr int kTokBuckets = 256;  // select_top_keys histogram (fewer buckets than the bit-pattern select of
                                  // the two-level route: equal score intervals keep the boundary small)
constexpr int kTokRankCap = 128;  // boundary keys ranked pairwise in select_top_keys
constexpr int kTokRefine = 9;     // key-range refinements (each shrinks a 64-bit range ~256x: 8 suffice)

// dot8 with one packed fp32 FMA per bf16 pair: even elements accumulate in .x,
// odd ones in .y, each rounding exactly like the scalar fmaf chain of dot8.
__device__ __forceinline__ float dot8_x2(const uint4 x, const float (&q)[8]) {
  float2 s = __fmul2_rn(make_float2(bf16_lo(x.x), bf16_hi(x.x)), make_float2(q[0], q[1]));
  s = __ffma2_rn(make_float2(bf16_lo(x.y), bf16_hi(x.y)), make_float2(q[2], q[3]), s);
  s = __ffma2_rn(make_float2(bf16_lo(x.z), bf16_hi(x.z)), make_float2(q[4], q[5]), s);
  s = __ffma2_rn(make_float2(bf16_lo(x.w), bf16_hi(x.w)), make_float2(q[6], q[7]), s);
  return s.x + s.y;
}

// Score of a route key (inverse of float_order_bits on the upper word).
__device__ __forceinline__ float route_key_score(uint64_t key) {
  const uint32_t u = (uint32_t)(key >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// Top r of n distinct route keys (1 <= r < n), written to sel[] as their ids in
// the keys' storage order (the token keys are stored in ascending position, so
// the kept positions come out ascending). lo and hi are the least and greatest
// score among the keys. The first histogram cuts [lo, hi] into kTokBuckets equal
// score intervals, which for a bell-shaped score distribution leaves a few
// dozen keys in the bucket holding the r-th key whatever r is (cutting the
// order-preserving bit pattern instead crowds most keys into the few buckets
// of the typical magnitude). While that boundary bucket holds more than
// kTokRankCap keys, its key range is cut again into kTokBuckets equal intervals
// of the 64-bit key; the boundary keys are then ranked pairwise. Every bucket
// map is monotone in the key, so a bucket is a contiguous key range and the
// kept set equals a full sort's. kred: 2 * kRoutedWarps + 2 words.
__device__ __forceinline__ void select_top_keys(const uint64_t* keys, int n, int r, float lo, float hi, int* sel,
                                                  int* hist, int* misc, uint64_t* scratch, uint64_t* kred) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float vscale = hi > lo ? (float)kTokBuckets / (hi - lo) : 0.f;
  auto vbucket = [&](uint64_t key) {
    return min(kTokBuckets - 1, max(0, (int)((route_key_score(key) - lo) * vscale)));
  };
  // level 0: score buckets; level >= 1: key buckets inside [klo, khi]
  uint64_t klo = 0, khi = 0;
  float kscale = 0.f;
  int level = 0, need = r;
  auto member_bucket = [&](uint64_t key) -> int {
    if (level == 0) return vbucket(key);
    if (key < klo || key > khi) return -1;
    return min(kTokBuckets - 1, (int)((float)(key - klo) * kscale));
  };
  int bstar = 0, members = 0;
  if (tid == 0) kred[2 * kRoutedWarps] = ~0ull;  // kth; ordered by the first barrier below
  for (;;) {
    for (int i = tid; i < hist_index(kTokBuckets); i += kRoutedThreads) hist[i] = 0;
    if (tid == 0) {
      misc[0] = 0;
      misc[1] = 0;
      misc[2] = 0;
    }
    __syncthreads();
    for (int i = tid; i < n; i += kRoutedThreads) {
      const int bk = member_bucket(keys[i]);
      if (bk >= 0) atomicAdd(&hist[hist_index(bk)], 1);
    }
    __syncthreads();
    find_boundary_bucket<kTokBuckets>(hist, need, misc);
    __syncthreads();
    bstar = misc[0];
    need -= misc[1];
    members = hist[hist_index(bstar)];
    if (members <= kTokRankCap || level >= kTokRefine) break;
    // key range of the boundary bucket -> the next level's interval
    uint64_t mn = ~0ull, mx = 0ull;
    for (int i = tid; i < n; i += kRoutedThreads) {
      const uint64_t key = keys[i];
      if (member_bucket(key) == bstar) {
        mn = min(mn, key);
        mx = max(mx, key);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      mn = min(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
      mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    }
    if (lane == 0) {
      kred[2 * warp] = mn;
      kred[2 * warp + 1] = mx;
    }
    __syncthreads();
    klo = ~0ull;
    khi = 0ull;
#pragma unroll
    for (int w = 0; w < kRoutedWarps; ++w) {
      klo = min(klo, kred[2 * w]);
      khi = max(khi, kred[2 * w + 1]);
    }
    kscale = (float)kTokBuckets / ((float)(khi - klo) + 1.0f);
    ++level;
    __syncthreads();  // kred and misc are rewritten by the next level
  }
  // pairwise ranking of the boundary keys; kth = the need-th largest of them
  const bool in_scratch = members <= kTokRankCap;
  if (in_scratch) {
    for (int i = tid; i < n; i += kRoutedThreads) {
      const uint64_t key = keys[i];
      if (member_bucket(key) == bstar) {
        const int slot = atomicAdd(&misc[2], 1);
        if (slot < kTokRankCap) scratch[slot] = key;
      }
    }
    __syncthreads();
    const int m = min(members, kTokRankCap);
    for (int j = tid; j < m; j += kRoutedThreads) {
      const uint64_t kj = scratch[j];
      int rank = 0;
      for (int l = 0; l < m; ++l) rank += scratch[l] > kj;
      if (rank == need - 1) kred[2 * kRoutedWarps] = kj;
    }
  } else {
    // not reached with distinct keys (each level shrinks the key range by about
    // kTokBuckets); ranks the boundary keys against every key
    for (int i = tid; i < n; i += kRoutedThreads) {
      const uint64_t ki = keys[i];
      if (member_bucket(ki) != bstar) continue;
      int rank = 0;
      for (int l = 0; l < n; ++l) rank += keys[l] > ki && member_bucket(keys[l]) == bstar;
      if (rank == need - 1) kred[2 * kRoutedWarps] = ki;
    }
  }
  __syncthreads();
  const uint64_t kth = kred[2 * kRoutedWarps];
  const int per = (n + kRoutedThreads - 1) / kRoutedThreads;
  const int s0 = min(n, tid * per), s1 = min(n, s0 + per);
  int cnt = 0;
  for (int i = s0; i < s1; ++i) cnt += keys[i] >= kth;
  int pos = block_exclusive_scan(cnt, misc + 24);
  for (int i = s0; i < s1; ++i)
    if (keys[i] >= kth && pos < r) sel[pos++] = (int)route_key_id(keys[i]);
}

// attend_tiles with the logits of every entry already computed: tile t of the
// staged V rows takes the logits of candidates ents[16t .. 16t+15] from lg
// ([candidate][8] floats, written earlier in this launch: plain loads) in the
// S^T fragment layout of qk_fragments, then runs the same softmax update and PV.
template <int D>
__device__ __forceinline__ void attend_tiles_logits(AttnState<D>& st, const uint32_t* rows, const int* ents,
                                                    int n_entries, int tile0, int stride, const uint16_t* V,
                                                    const float* lg, uint4* tile, float sl, int lane) {
  const int n_tiles = (n_entries + 15) >> 4;
  if (tile0 >= n_tiles) return;
  const int g = lane >> 2, t = lane & 3;
  auto fetch_logits = [&](int tl, float2& la, float2& lb) {
    const int ia = min(16 * tl + g, n_entries - 1), ib = min(16 * tl + g + 8, n_entries - 1);
    la = *reinterpret_cast<const float2*>(lg + (int64_t)ents[ia] * 8 + 2 * t);
    lb = *reinterpret_cast<const float2*>(lg + (int64_t)ents[ib] * 8 + 2 * t);
  };
  uint4 vr[TileGeom<D>::NLD];
  float2 la, lb;
  fetch_rows<D>(vr, rows + 16 * tile0, V, lane);
  fetch_logits(tile0, la, lb);
  for (int tl = tile0; tl < n_tiles; tl += stride) {
    const int nt = tl + stride;
    float s[4] = {la.x, la.y, lb.x, lb.y};
    store_rows<D>(tile, vr, lane);
    if (nt < n_tiles) {
      fetch_rows<D>(vr, rows + 16 * nt, V, lane);
      fetch_logits(nt, la, lb);
    }
    __syncwarp();
    uint32_t b0, b1;
    softmax_update<D>(st, s, n_entries - 16 * tl, sl, lane, b0, b1);
    pv<D>(st, tile, b0, b1, lane);
    __syncwarp();
  }
}

// Most candidate tokens of the token step over every length up to max_len:
// C + kcap*C + (last block and tail, < 2C), or every token when nf <= 2 (< 3C).
__host__ __device__ inline int hisa_tok_pad(int C, int kcap) { return (kcap + 3) * C; }

template <int D>
__global__ void __launch_bounds__(kRoutedThreads, 2) hisa_decode_kernel(const RoutedArgs a) {
  using TG = TileGeom<D>;
  constexpr int U = TG::U, RPI = TG::RPI, NLD = TG::NLD;
  static_assert(NLD == U / 2, "butterfly pairs NLD values over U lanes");
  extern __shared__ __align__(16) unsigned char hisa_smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int P = (int)cluster.num_blocks();
  const int cr = (int)cluster.block_rank();
  const int unit = blockIdx.x / P;
  const int hkv = a.kv.hkv;
  const int b = unit / hkv, h = unit % hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = lane % U, rsub = lane / U;

  const int C = a.C, k_tok = a.k_tok;
  const HisaSmem lay(D, a.n_pad, a.kcap, hisa_tok_pad(C, a.kcap), k_tok);
  float* qsum = reinterpret_cast<float*>(hisa_smem + lay.qsum);
  int* sel = reinterpret_cast<int*>(hisa_smem + lay.sel);
  int* pages = reinterpret_cast<int*>(hisa_smem + lay.pages);
  float* red_m = reinterpret_cast<float*>(hisa_smem + lay.red_m);
  float* red_l = reinterpret_cast<float*>(hisa_smem + lay.red_l);
  float* cta_o = reinterpret_cast<float*>(hisa_smem + lay.cta_o);
  float* cta_m = reinterpret_cast<float*>(hisa_smem + lay.cta_m);
  float* cta_l = reinterpret_cast<float*>(hisa_smem + lay.cta_l);
  uint4* qfrag = reinterpret_cast<uint4*>(hisa_smem + lay.qfrag);
  int* hist = reinterpret_cast<int*>(hisa_smem + lay.hist);
  int* misc = reinterpret_cast<int*>(hisa_smem + lay.misc);
  uint32_t* rows = reinterpret_cast<uint32_t*>(hisa_smem + lay.rows);
  int* tsel = reinterpret_cast<int*>(hisa_smem + lay.tsel);
  float* tmm = reinterpret_cast<float*>(hisa_smem + lay.tmm);
  uint64_t* kred = reinterpret_cast<uint64_t*>(hisa_smem + lay.kred);
  uint64_t* ckeys = reinterpret_cast<uint64_t*>(hisa_smem + lay.ckeys);
  uint64_t* tkeys = reinterpret_cast<uint64_t*>(hisa_smem + lay.tkeys);
  uint64_t* scratch = reinterpret_cast<uint64_t*>(hisa_smem + lay.scratch);
  float* red_o = reinterpret_cast<float*>(hisa_smem + lay.red_o);
  uint4* tile = reinterpret_cast<uint4*>(hisa_smem + lay.tiles) + warp * TG::kTileSlots;

  const bool paged = a.kv.page_table != nullptr;
  const int L = a.kv.length(b);
  const int nf = L / C;
  const bool dense = nf <= 2;
  const int n_cand = dense ? 0 : nf - 2;
  const int r = n_cand < a.k ? n_cand : a.k;
  const int tail0 = dense ? 0 : (nf - 1) * C;
  const int n_ct = dense ? L : C + r * C + (L - tail0);  // candidate tokens of the token step
  const uint16_t* qb = a.q + ((int64_t)b * a.hq + (int64_t)h * a.R) * D;

  // Peers write keys into this CTA's shared memory: every CTA of the cluster
  // must have started first (arrive now, wait before the first remote store).
  cluster_arrive_relaxed();
  if (paged) {
    // physical page of every page slot the context touches (page = chunk)
    const int n_slots = (L + C - 1) / C;
    for (int i = tid; i < n_slots; i += kRoutedThreads) {
      int page = __ldg(a.kv.page_table + (int64_t)b * a.kv.max_pages + i);
      if ((unsigned)page >= (unsigned)a.kv.num_pages) {
        report_error(kErrPage);
        page = 0;  // read a real page; results after a reported error are unspecified
      }
      pages[i] = page;
    }
    __syncthreads();
  }
  auto tok_row = [&](int t) -> uint32_t {
    if (!paged) return (uint32_t)(((int64_t)b * hkv + h) * a.kv.max_len + t);
    const int slot = t / C;  // page = chunk
    return (uint32_t)(((int64_t)pages[slot] * hkv + h) * C + (t - slot * C));
  };

  // ------------------------------------------------------------------ R1
  const bool select_needed = n_cand > r;
  {
    const int c0 = (int)((int64_t)n_cand * cr / P), c1 = (int)((int64_t)n_cand * (cr + 1) / P);
    const int n_rows = c1 - c0;
    const int nb = select_needed ? (n_rows + 15) / 16 : 0;
    float qv[8];
    auto issue = [&](int bi, uint4(&x)[NLD]) {
#pragma unroll
      for (int k = 0; k < NLD; ++k) {
        const int i = min(16 * bi + RPI * k + rsub, n_rows - 1);
        const int c = c0 + i + 1;
        x[k] = ldg_stream(a.sv.chunk + a.sv.chunk_off(paged, b, h, hkv, c, paged ? pages[c] : 0) + 8 * u);
      }
    };
    auto consume = [&](int bi, const uint4(&x)[NLD]) {
      float v[NLD];
#pragma unroll
      for (int k = 0; k < NLD; ++k) v[k] = dot8_x2(x[k], qv);
      int idx;
      const float score = butterfly_sum<NLD>(v, lane, idx);
      const int i = 16 * bi + RPI * idx + rsub;
      if ((lane & 1) == 0 && i < n_rows) {
        const int cand = c0 + i;
        const uint64_t key = route_key(score, (uint32_t)(cand + 1));
        for (int pr = 0; pr < P; ++pr) cluster.map_shared_rank(ckeys, pr)[cand] = key;
      }
    };
    uint4 xa[NLD], xb[NLD];
    if (warp < nb) issue(warp, xa);
    if (warp + kRoutedWarps < nb) issue(warp + kRoutedWarps, xb);
    for (int e = tid; e < D; e += kRoutedThreads) {
      float sq = 0.f;
      for (int i = 0; i < a.R; ++i) sq += bf16_to_f(qb[(int64_t)i * D + e]);
      qsum[e] = sq;
    }
    stage_q_fragments<D>(qfrag, qb, a.R, tid, kRoutedThreads);
    __syncthreads();
    cluster_wait();
    if (nb > 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j) qv[j] = qsum[8 * u + j];
      for (int bi = warp; bi < nb; bi += 2 * kRoutedWarps) {
        consume(bi, xa);
        if (bi + 2 * kRoutedWarps < nb) issue(bi + 2 * kRoutedWarps, xa);
        if (bi + kRoutedWarps < nb) {
          consume(bi + kRoutedWarps, xb);
          if (bi + 3 * kRoutedWarps < nb) issue(bi + 3 * kRoutedWarps, xb);
        }
      }
    }
  }
  cluster.sync();

  // ------------------------------------------------------------------ R2
  if (select_needed) {
    select_top_chunks<kChunkBuckets>(ckeys, n_cand, r, sel, hist, misc, scratch, kDecodeScratchKeys);
  } else {
    for (int i = tid; i < r; i += kRoutedThreads) sel[i] = i + 1;
  }
  __syncthreads();

  // candidate e of the token step -> token position (ascending in e)
  auto cand_tok = [&](int e) -> int {
    if (dense || e < C) return e;
    const int v = e - C;
    if (v < r * C) return sel[v / C] * C + (v - (v / C) * C);
    return tail0 + (v - r * C);
  };

  // ------------------------------------------------------------- T1 + T2
  const bool keep_all = n_ct <= k_tok;
  if (!keep_all) {
    // 16-candidate batches split over the CTAs. C % 16 == 0, so a batch never
    // straddles two segments (first chunk, a kept chunk, last chunk + tail):
    // its 16 positions are consecutive and lie in one page, one contiguous run
    // of K rows that the warp reads with whole-row coalesced loads.
    const int nbt = (n_ct + 15) / 16;
    const int bb0 = (int)((int64_t)nbt * cr / P), bb1 = (int)((int64_t)nbt * (cr + 1) / P);
    const int nb = bb1 - bb0;
    auto batch_tok = [&](int bi) -> int {  // position of candidate 16 * bi
      const int e0 = 16 * bi;
      if (dense) return e0;
      const int sg = e0 / C;
      if (sg == 0) return e0;
      if (sg <= r) return sel[sg - 1] * C + (e0 - sg * C);
      return tail0 + (e0 - (r + 1) * C);
    };
    float qv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) qv[j] = qsum[8 * u + j];
    float smin = __int_as_float(0x7f800000), smax = -__int_as_float(0x7f800000);
    // key of candidate e: its score, then the lower candidate index first (the
    // candidates are in ascending position, so this is the lower position)
    auto emit_key = [&](int e, float score) {
      const uint64_t key = route_key(score, (uint32_t)e);
      smin = fminf(smin, score);
      smax = fmaxf(smax, score);
      if (P == 1) {
        tkeys[e] = key;
      } else {
        for (int pr = 0; pr < P; ++pr) cluster.map_shared_rank(tkeys, pr)[e] = key;
      }
    };
    // issue returns the batch's first position (unused by consume)
    auto issue = [&](int j, uint4(&x)[NLD]) -> int {
      const int bi = bb0 + j;
      const int nv = min(16, n_ct - 16 * bi);
      const int t0 = batch_tok(bi);
      const uint16_t* src = a.kv.k + (int64_t)tok_row(t0) * D + 8 * u;
      if (nv == 16) {
#pragma unroll
        for (int k = 0; k < NLD; ++k) x[k] = ldg_stream(src + (RPI * k + rsub) * D);
      } else {
#pragma unroll
        for (int k = 0; k < NLD; ++k) x[k] = ldg_stream(src + min(RPI * k + rsub, nv - 1) * D);
      }
      return t0;
    };
    auto consume = [&](int j, const uint4(&x)[NLD], int /* first position */) {
      const int bi = bb0 + j;
      float v[NLD];
#pragma unroll
      for (int k = 0; k < NLD; ++k) v[k] = dot8_x2(x[k], qv);
      int idx;
      const float score = butterfly_sum<NLD>(v, lane, idx);
      const int i = RPI * idx + rsub;
      if ((lane & 1) == 0 && i < n_ct - 16 * bi) emit_key(16 * bi + i, score);
    };
    if (a.logits == nullptr) {
      uint4 xa[NLD], xb[NLD];
      int ta = 0, tb = 0;
      if (warp < nb) ta = issue(warp, xa);
      if (warp + kRoutedWarps < nb) tb = issue(warp + kRoutedWarps, xb);
      for (int j = warp; j < nb; j += 2 * kRoutedWarps) {
        consume(j, xa, ta);
        if (j + 2 * kRoutedWarps < nb) ta = issue(j + 2 * kRoutedWarps, xa);
        if (j + kRoutedWarps < nb) {
          consume(j + kRoutedWarps, xb, tb);
          if (j + 3 * kRoutedWarps < nb) tb = issue(j + 3 * kRoutedWarps, xb);
        }
      }
    } else {
      // QK^T tiles: lane (g, t) loads unit t + 4j of the batch's rows g and g+8
      // (64 contiguous bytes of each row per warp instruction); the score of a
      // token is the sum over the query heads of its logits (padding heads have
      // zero queries), reduced over the four lanes that share the token
      constexpr int KJ = TG::KJ;
      float* lg = a.logits + (int64_t)unit * a.lg_stride;
      const int gq = lane >> 2, tq = lane & 3;
      auto issue_mma = [&](int j, uint4(&ka)[KJ], uint4(&kb)[KJ]) {
        const int bi = bb0 + j;
        const int nv = min(16, n_ct - 16 * bi);
        const uint16_t* src = a.kv.k + (int64_t)tok_row(batch_tok(bi)) * D + 8 * tq;
        const int ra = min(gq, nv - 1), rb = min(gq + 8, nv - 1);
#pragma unroll
        for (int jj = 0; jj < KJ; ++jj) {
          ka[jj] = ldg_stream(src + (int64_t)ra * D + 32 * jj);
          kb[jj] = ldg_stream(src + (int64_t)rb * D + 32 * jj);
        }
      };
      auto consume_mma = [&](int j, const uint4(&ka)[KJ], const uint4(&kb)[KJ]) {
        const int bi = bb0 + j;
        const int nv = min(16, n_ct - 16 * bi);
        float sv[4];
        qk_fragments<D>(sv, ka, kb, qfrag, lane);
        float sa = sv[0] + sv[1], sb = sv[2] + sv[3];
        sa += __shfl_xor_sync(0xFFFFFFFFu, sa, 1);
        sb += __shfl_xor_sync(0xFFFFFFFFu, sb, 1);
        sa += __shfl_xor_sync(0xFFFFFFFFu, sa, 2);
        sb += __shfl_xor_sync(0xFFFFFFFFu, sb, 2);
        const int ea = 16 * bi + gq, eb = ea + 8;
        if (gq < nv) *reinterpret_cast<float2*>(lg + (int64_t)ea * 8 + 2 * tq) = make_float2(sv[0], sv[1]);
        if (gq + 8 < nv) *reinterpret_cast<float2*>(lg + (int64_t)eb * 8 + 2 * tq) = make_float2(sv[2], sv[3]);
        if (tq == 0) {
          if (gq < nv) emit_key(ea, sa);
          if (gq + 8 < nv) emit_key(eb, sb);
        }
      };
      uint4 ka0[KJ], kb0[KJ], ka1[KJ], kb1[KJ];
      if (warp < nb) issue_mma(warp, ka0, kb0);
      if (warp + kRoutedWarps < nb) issue_mma(warp + kRoutedWarps, ka1, kb1);
      for (int j = warp; j < nb; j += 2 * kRoutedWarps) {
        consume_mma(j, ka0, kb0);
        if (j + 2 * kRoutedWarps < nb) issue_mma(j + 2 * kRoutedWarps, ka0, kb0);
        if (j + kRoutedWarps < nb) {
          consume_mma(j + kRoutedWarps, ka1, kb1);
          if (j + 3 * kRoutedWarps < nb) issue_mma(j + 3 * kRoutedWarps, ka1, kb1);
        }
      }
    }
    publish_range(smin, smax, tmm, kTmmTok, cluster, P, cr);
    cluster.sync();
    float lo, hi;
    cluster_range(tmm, kTmmTok, P, lo, hi);
    // top k_tok of the n_ct keys, as candidate indices in ascending order (so
    // the kept positions come out ascending)
    select_top_keys(tkeys, n_ct, k_tok, lo, hi, tsel, hist, misc, scratch, kred);
    __syncthreads();
  }
  const int S = keep_all ? n_ct : k_tok;
  auto entry_tok = [&](int e) -> int { return cand_tok(keep_all ? e : tsel[e]); };

  // ------------------------------------------------------------------- A
  const int n_tiles = (S + 15) / 16;
  const int t0 = (int)((int64_t)n_tiles * cr / P), t1 = (int)((int64_t)n_tiles * (cr + 1) / P);
  const int e_begin = 16 * t0, e_end = min(16 * t1, S);
  if (a.idx_out != nullptr) {
    const int cap = min(S, a.idx_stride);
    if (S > a.idx_stride && tid == 0 && cr == 0) report_error(kErrIndex);
    for (int e = e_begin + tid; e < min(e_end, cap); e += kRoutedThreads)
      a.idx_out[(int64_t)unit * a.idx_stride + e] = entry_tok(e);
    if (cr == 0 && tid == 0) a.n_idx_out[unit] = S;
  }
  AttnState<D> st;
  st.init();
  for (int eb = e_begin; eb < e_end; eb += kEntryBatch) {
    const int n_e = min(kEntryBatch, e_end - eb);
    const int n_t = (n_e + 15) / 16;
    __syncthreads();  // the previous batch's tiles are done with rows[]
    // padding entries of the last tile read the batch's first row (masked)
    for (int i = tid; i < n_t * 16; i += kRoutedThreads) rows[i] = tok_row(entry_tok(eb + (i < n_e ? i : 0)));
    __syncthreads();
    if (a.logits != nullptr && !keep_all)
      attend_tiles_logits<D>(st, rows, tsel + eb, n_e, warp, kRoutedWarps, a.kv.v,
                             a.logits + (int64_t)unit * a.lg_stride, tile, a.scale_log2, lane);
    else
      attend_tiles<D>(st, rows, n_e, warp, kRoutedWarps, a.kv.k, a.kv.v, qfrag, tile, a.scale_log2, lane);
  }
  finish_attention<D>(st, a, cluster, P, cr, b, h, red_o, red_m, red_l, cta_o, cta_m, cta_l);
}

}  // namespace hga
