// Balanced decode in two kernels: route once, then attend equal slices of all
// routed tiles (group sizes that are a whole number of 16-token tiles).
//
// "Hierarchical Global Attention (HGA)", abstract: pick chunks by their
// summaries, then the best groups inside the picked chunks, then attend exactly
// over the picked tokens; the first chunk (sink) and the last chunk plus the
// partial tail (local) are always kept (HISA article, two-step block filter).
//
// Why two kernels. The fused decode kernel gives each (sequence, KV head) unit
// one cluster, so the work per SM follows the unit count: 256 units on 148 SMs
// leave some SMs with one unit and others with two, and 64 units leave most of
// the machine idle during the serial routing prologue. Here the number of tiles
// of every unit is known from its length alone (sink and local tiles, plus
// top-k chunks x top-G groups x g/16 tiles), so the attention kernel can cut the
// concatenation of all units' tiles into equal slices, one per CTA, before any
// routing result exists:
//
//   route_tiles_kernel   one cluster of P CTAs per unit: chunk scores (the
//       head-summed query against the candidate chunk summaries, keys to every
//       CTA of the cluster through DSMEM), the bucket select of the top-k chunk
//       ids, then the group scores of this CTA's share of the kept chunks and
//       their top-G masks; it writes the first K/V row of every routed tile
//       (and, on request, the routed positions). It also clears the unit's
//       merge counter and lets the attention kernel launch early
//       (griddepcontrol.launch_dependents).
//   balanced_attend_kernel  a grid of 2 CTAs per SM (or fewer for small
//       problems); CTA c attends tiles [c T / G, (c + 1) T / G) of the T tiles
//       of all units, in unit order, sink and local tiles of a unit first. The
//       sink and local tiles need no routing, so a CTA attends those before it
//       waits for the route kernel (griddepcontrol.wait). A CTA that holds a
//       whole unit writes its output; the CTAs that share a unit leave their
//       partial softmax state (o, running max, denominator) in the workspace,
//       and the last of them to finish (an atomic count per unit) merges the
//       partials and writes the output. No CTA waits for another.
#pragma once

#include "hga_decode.cuh"

namespace hga {

// Programmatic dependent launch (PTX griddepcontrol): the dependent grid may
// start once every CTA of the primary grid has executed launch_dependents (or
// exited); wait blocks until the primary grid has completed and its memory is
// visible. Both are no-ops for a grid launched without the dependency.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

constexpr int kSplitMaxBatch = 4096;            // sequences the attention kernel's prefix table holds
constexpr int kPartFloats = kMaxHeadsPerKv * 130;  // o[8][128], m[8], l[8] (+ padding) per partial slot

struct SplitArgs {
  uint32_t* tiles;  // [units][tile_stride]: first K/V row of every routed tile, in list order
  int tile_stride;  // >= kcap * top_groups * (group / 16)
  float* part;      // [grid + units][kPartFloats] partial softmax states (slot = CTA + unit)
  int* count;       // [units] partials merged so far (cleared by the route kernel)
  int grid;         // CTAs of the attention kernel
};

// Tiles of one unit at context length L (the same on host and device): the sink
// and local-plus-tail tiles (n_fixed), then r routed chunks x G groups x g/16.
struct UnitTiles {
  int n_fixed, n_routed, r, tail0;
  bool dense;
  __host__ __device__ UnitTiles(int L, int C, int g, int k, int G) {
    const int nf = L / C;
    dense = nf <= 2;
    if (dense) {
      n_fixed = (L + 15) / 16;
      n_routed = r = tail0 = 0;
    } else {
      r = nf - 2 < k ? nf - 2 : k;
      tail0 = (nf - 1) * C;
      n_fixed = C / 16 + (L - tail0 + 15) / 16;
      n_routed = r * G * (g / 16);
    }
  }
  __host__ __device__ int total() const { return n_fixed + n_routed; }
};

// Shared-memory carve-up of the route kernel (byte offsets, host and device).
struct RouteTilesSmem {
  int qsum, sel, pages, hist, misc, gmask, gsc, keys, scratch, total;
  __host__ __device__ static int up16(int x) { return (x + 15) & ~15; }
  __host__ __device__ RouteTilesSmem(int D, int n_pad, int kcap, int gpc) {
    int o = 0;
    qsum = o;    o = up16(o + 4 * D);
    sel = o;     o = up16(o + 4 * kcap);
    pages = o;   o = up16(o + 4 * (n_pad + 4));
    hist = o;    o = up16(o + 4 * kHistWords);
    misc = o;    o = up16(o + 4 * 32);
    gmask = o;   o = up16(o + 4 * kcap);
    gsc = o;     o = up16(o + 4 * kcap * gpc);
    keys = o;    o = up16(o + 8 * n_pad);
    scratch = o; o = up16(o + 8 * kDecodeScratchKeys);
    total = o;
  }
};

// Head-summed scores of n_rows summary rows (row i at row_ptr(i)), streamed by
// the CTA's warps in 16-row register batches with two batches in flight per
// warp: every lane loads whole-row 16-byte units, dots them with its slice of
// the head-summed query, and a halving butterfly leaves row i's score on one
// lane pair, handed to emit(i, score) by the even lane. start() issues the
// first two batches (before the query sum exists); finish() needs qsum.
template <int D>
struct RowScorer {
  static constexpr int U = TileGeom<D>::U, RPI = TileGeom<D>::RPI, NLD = TileGeom<D>::NLD;
  uint4 xa[NLD], xb[NLD];
  int n_rows, nb, warp, lane;

  template <typename RowPtr>
  __device__ __forceinline__ void issue(int bi, uint4 (&x)[NLD], RowPtr row_ptr) {
    const int u = lane % U, rsub = lane / U;
#pragma unroll
    for (int k = 0; k < NLD; ++k) {
      const int i = min(16 * bi + RPI * k + rsub, n_rows - 1);
      x[k] = ldg_stream(row_ptr(i) + 8 * u);
    }
  }
  template <typename Emit>
  __device__ __forceinline__ void consume(int bi, const uint4 (&x)[NLD], const float (&qv)[8], Emit emit) {
    float v[NLD];
#pragma unroll
    for (int k = 0; k < NLD; ++k) v[k] = dot8(x[k], qv);
    int idx;
    const float score = butterfly_sum<NLD>(v, lane, idx);
    const int i = 16 * bi + RPI * idx + lane / U;
    if ((lane & 1) == 0 && i < n_rows) emit(i, score);
  }
  template <typename RowPtr>
  __device__ __forceinline__ void start(int rows, RowPtr row_ptr) {
    warp = threadIdx.x >> 5;
    lane = threadIdx.x & 31;
    n_rows = rows;
    nb = (rows + 15) / 16;
    if (warp < nb) issue(warp, xa, row_ptr);
    if (warp + kRoutedWarps < nb) issue(warp + kRoutedWarps, xb, row_ptr);
  }
  template <typename RowPtr, typename Emit>
  __device__ __forceinline__ void finish(const float* qsum, RowPtr row_ptr, Emit emit) {
    if (nb == 0) return;
    float qv[8];
    const int u = lane % U;
#pragma unroll
    for (int j = 0; j < 8; ++j) qv[j] = qsum[8 * u + j];
    for (int bi = warp; bi < nb; bi += 2 * kRoutedWarps) {
      consume(bi, xa, qv, emit);
      if (bi + 2 * kRoutedWarps < nb) issue(bi + 2 * kRoutedWarps, xa, row_ptr);
      if (bi + kRoutedWarps < nb) {
        consume(bi + kRoutedWarps, xb, qv, emit);
        if (bi + 3 * kRoutedWarps < nb) issue(bi + 3 * kRoutedWarps, xb, row_ptr);
      }
    }
  }
};

template <int D>
__global__ void __launch_bounds__(kRoutedThreads, 2) route_tiles_kernel(const RoutedArgs a, const SplitArgs sp) {
  extern __shared__ __align__(16) unsigned char rt_smem[];
  // the attention kernel may take free SM slots now; it waits for this grid
  // before it reads anything written here
  griddep_launch_dependents();
  cg::cluster_group cluster = cg::this_cluster();
  const int P = (int)cluster.num_blocks();
  const int cr = (int)cluster.block_rank();
  const int unit = blockIdx.x / P;
  const int hkv = a.kv.hkv;
  const int b = unit / hkv, h = unit % hkv;
  const int tid = threadIdx.x;

  const int C = a.C, g = a.g, gpc = C / g, gk = a.G;
  const RouteTilesSmem lay(D, a.n_pad, a.kcap, gpc);
  float* qsum = reinterpret_cast<float*>(rt_smem + lay.qsum);
  int* sel = reinterpret_cast<int*>(rt_smem + lay.sel);
  int* pages = reinterpret_cast<int*>(rt_smem + lay.pages);
  int* hist = reinterpret_cast<int*>(rt_smem + lay.hist);
  int* misc = reinterpret_cast<int*>(rt_smem + lay.misc);
  uint32_t* gmask = reinterpret_cast<uint32_t*>(rt_smem + lay.gmask);
  float* gsc = reinterpret_cast<float*>(rt_smem + lay.gsc);
  uint64_t* keys = reinterpret_cast<uint64_t*>(rt_smem + lay.keys);
  uint64_t* scratch = reinterpret_cast<uint64_t*>(rt_smem + lay.scratch);

  const bool paged = a.kv.page_table != nullptr;
  const int L = a.kv.length(b);
  const UnitTiles ut(L, C, g, a.k, gk);
  const int nf = L / C;
  const int n_cand = ut.dense ? 0 : nf - 2;
  const int r = ut.r;
  const uint16_t* qb = a.q + ((int64_t)b * a.hq + (int64_t)h * a.R) * D;

  // peers write keys into this CTA's shared memory in R1 (arrive now, wait
  // before the first remote store)
  cluster_arrive_relaxed();
  if (paged) {
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

  // R1: this CTA's share of candidates 1..nf-2, first loads before the query sum
  const bool select_needed = n_cand > r;
  const int c0 = (int)((int64_t)n_cand * cr / P), c1 = (int)((int64_t)n_cand * (cr + 1) / P);
  auto chunk_row = [&](int i) -> const uint16_t* {
    const int c = c0 + i + 1;
    return a.sv.chunk + a.sv.chunk_off(paged, b, h, hkv, c, paged ? pages[c] : 0);
  };
  RowScorer<D> r1;
  r1.start(select_needed ? c1 - c0 : 0, chunk_row);
  for (int e = tid; e < D; e += kRoutedThreads) {
    float sq = 0.f;
    for (int i = 0; i < a.R; ++i) sq += bf16_to_f(qb[(int64_t)i * D + e]);
    qsum[e] = sq;
  }
  __syncthreads();
  cluster_wait();
  r1.finish(qsum, chunk_row, [&](int i, float score) {
    const int cand = c0 + i;
    const uint64_t key = route_key(score, (uint32_t)(cand + 1));
    for (int pr = 0; pr < P; ++pr) cluster.map_shared_rank(keys, pr)[cand] = key;
  });
  // after this barrier no CTA touches another's shared memory
  cluster.sync();

  // R2: top-r chunk ids, ascending
  if (select_needed) {
    select_top_chunks(keys, n_cand, r, sel, hist, misc, scratch, kDecodeScratchKeys);
  } else {
    for (int i = tid; i < r; i += kRoutedThreads) sel[i] = i + 1;
  }
  __syncthreads();

  // R3: group scores of this CTA's kept chunks [s0, s1), then top-G masks
  const bool all_groups = gk >= gpc;
  const int s0 = (int)((int64_t)r * cr / P), s1 = (int)((int64_t)r * (cr + 1) / P);
  const int nk = s1 - s0;
  if (!all_groups && nk > 0) {
    auto group_row = [&](int i) -> const uint16_t* {
      const int ci = i / gpc, j = i - ci * gpc;
      const int c = sel[s0 + ci];
      return a.sv.group + a.sv.group_off(paged, b, h, hkv, c, paged ? pages[c] : 0) + (int64_t)j * D;
    };
    for (int i = tid; i < nk; i += kRoutedThreads) gmask[i] = 0u;
    RowScorer<D> r3;
    r3.start(nk * gpc, group_row);
    r3.finish(qsum, group_row, [&](int i, float score) { gsc[i] = score; });
    __syncthreads();
    for (int i = tid; i < nk * gpc; i += kRoutedThreads) {
      const int ci = i / gpc, j = i - ci * gpc;
      const float tj = gsc[i];
      const float* row_scores = gsc + ci * gpc;
      int rank = 0;
      for (int l = 0; l < gpc; ++l) {
        const float tl = row_scores[l];
        rank += (tl > tj) || (tl == tj && l < j);
      }
      if (rank < gk) atomicOr(&gmask[ci], 1u << j);
    }
    __syncthreads();
  }

  // first K/V row of every routed tile of this CTA's chunks (list order: kept
  // chunks ascending, groups ascending inside a chunk, 16-token tiles inside a group)
  const uint32_t full_mask = gpc >= 32 ? 0xFFFFFFFFu : ((1u << gpc) - 1u);
  const int gsel = all_groups ? gpc : gk;
  const int gt = g / 16, JT = gsel * gt, span = gsel * g;
  auto tok_row = [&](int t0) -> uint32_t {
    if (!paged) return (uint32_t)(((int64_t)b * hkv + h) * a.kv.max_len + t0);
    const int slot = t0 / C;  // page = chunk
    return (uint32_t)(((int64_t)pages[slot] * hkv + h) * C + (t0 - slot * C));
  };
  auto nth_group = [&](int ci_local, int gr) -> int {
    uint32_t m = all_groups ? full_mask : gmask[ci_local];
    for (int x = 0; x < gr; ++x) m &= m - 1;
    return m ? __ffs(m) - 1 : 0;
  };
  uint32_t* trow = sp.tiles + (int64_t)unit * sp.tile_stride;
  for (int e = tid; e < nk * JT; e += kRoutedThreads) {
    const int cl = e / JT, tt = e - cl * JT;
    const int gr = tt / gt, sub = tt - gr * gt;
    const int c = sel[s0 + cl];
    trow[(s0 + cl) * JT + tt] = tok_row(c * C + nth_group(cl, gr) * g + 16 * sub);
  }

  // routed positions (optional), ascending: sink, kept groups, local + tail
  if (a.idx_out != nullptr) {
    const int S = ut.dense ? L : C + r * span + (L - ut.tail0);
    int32_t* idx_row = a.idx_out + (int64_t)unit * a.idx_stride;
    const int cap = S < a.idx_stride ? S : a.idx_stride;
    if (S > a.idx_stride && tid == 0 && cr == 0) report_error(kErrIndex);
    for (int e = tid; e < nk * span; e += kRoutedThreads) {
      const int cl = e / span, w = e - cl * span, gr = w / g;
      const int entry = C + (s0 + cl) * span + w;
      if (entry < cap) idx_row[entry] = sel[s0 + cl] * C + nth_group(cl, gr) * g + (w - gr * g);
    }
    // fixed entries (sink, local + tail; or the whole dense context), split over the cluster
    const int n_fixed_tok = ut.dense ? L : C + (L - ut.tail0);
    for (int e = cr * kRoutedThreads + tid; e < n_fixed_tok; e += P * kRoutedThreads) {
      const int entry = (ut.dense || e < C) ? e : e + r * span;
      const int tok = (ut.dense || e < C) ? e : ut.tail0 + (e - C);
      if (entry < cap) idx_row[entry] = tok;
    }
    if (cr == 0 && tid == 0) a.n_idx_out[unit] = S;
  }
  if (cr == 0 && tid == 0) sp.count[unit] = 0;
}

// Shared-memory carve-up of the attention kernel (byte offsets, host and device).
struct BalancedSmem {
  int qfrag, red_m, red_l, misc, prefix, uni, tiles, red_o, total;
  __host__ __device__ static int up16(int x) { return (x + 15) & ~15; }
  __host__ __device__ BalancedSmem(int D, int batch, int grid) {
    int o = 0;
    qfrag = o;  o = up16(o + 16 * 32 * (D / 32));
    red_m = o;  o = up16(o + 4 * kRoutedWarps * kMaxHeadsPerKv);
    red_l = o;  o = up16(o + 4 * kRoutedWarps * kMaxHeadsPerKv);
    misc = o;   o = up16(o + 4 * 32);
    prefix = o; o = up16(o + 4 * (batch + 1));
    // union: per-warp K/V tiles while attending | per-warp partial outputs
    uni = o;
    tiles = o;
    red_o = o;
    int u = kRoutedWarps * 16 * D * 2;
    const int red_bytes = 4 * kRoutedWarps * kMaxHeadsPerKv * D;
    if (red_bytes > u) u = red_bytes;
    const int merge_bytes = 2 * 4 * kMaxHeadsPerKv * grid;  // weights and denominators of <= grid partials
    if (merge_bytes > u) u = merge_bytes;
    o = up16(o + u);
    total = o;
  }
};

// CTA of tile t when T tiles are cut into G <= T equal slices [c T / G, (c + 1) T / G)
// (the largest c whose slice starts at or before t).
__device__ __forceinline__ int slice_of(int64_t t, int64_t T, int G) {
  return (int)(((t + 1) * G - 1) / T);
}

template <int D>
__global__ void __launch_bounds__(kRoutedThreads, 2) balanced_attend_kernel(const RoutedArgs a, const SplitArgs sp) {
  using TG = TileGeom<D>;
  constexpr int U = TG::U, RPI = TG::RPI, NLD = TG::NLD;
  extern __shared__ __align__(16) unsigned char ba_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u_lane = lane % U, rsub = lane / U;
  const BalancedSmem lay(D, a.kv.batch, sp.grid);
  uint4* qfrag = reinterpret_cast<uint4*>(ba_smem + lay.qfrag);
  float* red_m = reinterpret_cast<float*>(ba_smem + lay.red_m);
  float* red_l = reinterpret_cast<float*>(ba_smem + lay.red_l);
  int* misc = reinterpret_cast<int*>(ba_smem + lay.misc);
  int* prefix = reinterpret_cast<int*>(ba_smem + lay.prefix);
  float* red_o = reinterpret_cast<float*>(ba_smem + lay.red_o);
  uint4* tile = reinterpret_cast<uint4*>(ba_smem + lay.tiles) + warp * TG::kTileSlots;

  const int B = a.kv.batch, hkv = a.kv.hkv, C = a.C;
  const int G = sp.grid, c = blockIdx.x;
  const bool paged = a.kv.page_table != nullptr;

  // tiles per sequence (every KV head of a sequence has the same count), and the
  // prefix over sequences of hkv * tiles: unit (b, h) starts at prefix[b] + h * tiles(b)
  {
    const int per = (B + kRoutedThreads - 1) / kRoutedThreads;
    const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
    int sum = 0;
    for (int bb = b0; bb < b1; ++bb) {
      const int Lb = a.kv.length(bb);
      sum += hkv * UnitTiles(Lb, C, a.g, a.k, a.G).total();
    }
    int pos = block_exclusive_scan(sum, misc + 24);
    for (int bb = b0; bb < b1; ++bb) {
      prefix[bb] = pos;
      pos += hkv * UnitTiles(a.kv.length(bb), C, a.g, a.k, a.G).total();
    }
    if (b1 == B && b0 < b1) prefix[B] = pos;  // the thread holding the last sequence (B >= 1)
  }
  __syncthreads();
  const int64_t T = prefix[B];
  // Ge = min(G, T) slices, so that no slice is empty and every CTA between the
  // first and the last of a unit's slices holds a part of it; CTAs c >= Ge idle
  const int Ge = T < G ? (int)T : G;
  const int64_t t0 = c < Ge ? T * c / Ge : T, t1 = c < Ge ? T * (c + 1) / Ge : T;
  const int last_cta = Ge > 0 ? Ge - 1 : 0;

  AttnState<D> st;
  bool waited = false;
  auto wait_route = [&]() {
    if (!waited) {
      griddep_wait();
      waited = true;
    }
  };

  // sequences whose units this CTA may touch start at the first b whose tiles
  // end at or after t0 (that also reaches empty sequences starting at t0)
  int bfirst = 0;
  {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid + 1] >= t0) hi = mid; else lo = mid + 1;
    }
    bfirst = lo;
  }
  // rows of the K/V buffers (bound for the tile rows the route kernel left in the workspace)
  const int64_t n_rows_kv = paged ? (int64_t)a.kv.num_pages * hkv * a.kv.page_size
                                  : (int64_t)B * hkv * a.kv.max_len;
  for (int b = bfirst; b < B && prefix[b] <= t1; ++b) {
    const int L = a.kv.length(b);
    const UnitTiles ut(L, C, a.g, a.k, a.G);
    const int nt = ut.total();
    const uint16_t* Kp = a.kv.k;
    const uint16_t* Vp = a.kv.v;
    for (int h = 0; h < hkv; ++h) {
      const int unit = b * hkv + h;
      const int64_t U0 = prefix[b] + (int64_t)h * nt, U1 = U0 + nt;
      if (nt == 0) {
        // an empty unit belongs to the CTA whose slice holds its start position
        const bool mine = (U0 >= t0 && U0 < t1) || (U0 == T && c == last_cta);
        if (mine) {
          for (int i = tid; i < a.R * D; i += kRoutedThreads) {
            const int n = i / D, dd = i - n * D;
            const int64_t head = (int64_t)b * a.hq + (int64_t)h * a.R + n;
            a.out[head * D + dd] = 0.f;
            if (dd == 0 && a.lse != nullptr) a.lse[head] = -INFINITY;
          }
        }
        continue;
      }
      if (U1 <= t0) continue;
      if (U0 >= t1) break;
      const int k0 = (int)((U0 >= t0 ? U0 : t0) - U0), k1 = (int)((U1 <= t1 ? U1 : t1) - U0);
      const bool whole = U0 >= t0 && U1 <= t1;
      if (k1 > ut.n_fixed) wait_route();  // the segment reaches the routed tiles

      __syncthreads();  // the previous unit's readers of qfrag / red_* are done
      stage_q_fragments<D>(qfrag, a.q + ((int64_t)b * a.hq + (int64_t)h * a.R) * D, a.R, tid, kRoutedThreads);
      __syncthreads();
      st.init();

      const uint32_t* trow = sp.tiles + (int64_t)unit * sp.tile_stride;
      // this warp's tiles are k = first + W q (q = 0, 1, ...); the rows of its
      // routed tiles are read 32 at a time, one per lane, so that a tile's gather
      // does not wait for a load of its row index
      const int first = k0 + warp;
      uint32_t lane_row = 0;
      int row_block = -1;
      auto tile_at = [&](int k) -> TileRef {
        TileRef t;
        if (k < ut.n_fixed) {
          const int t_0 = (ut.dense || k < C / 16) ? 16 * k : ut.tail0 + 16 * (k - C / 16);
          t.nvalid = min(16, L - t_0);
          if (!paged) {
            t.row0 = (uint32_t)(((int64_t)b * hkv + h) * a.kv.max_len + t_0);
          } else {
            const uint32_t r0 = a.kv.row(b, h, t_0);  // validates the page id
            t.row0 = r0 == kInvalidRow ? 0u : r0;
          }
        } else {
          const int q = (k - first) / kRoutedWarps;
          if ((q >> 5) != row_block) {  // warp-uniform: every lane asks for the same q
            row_block = q >> 5;
            const int kk = first + kRoutedWarps * (32 * row_block + lane);
            lane_row = (kk < k1 && kk >= ut.n_fixed) ? __ldcg(trow + (kk - ut.n_fixed)) : 0u;
          }
          t.row0 = __shfl_sync(0xFFFFFFFFu, lane_row, q & 31);
          t.nvalid = 16;
          if ((int64_t)t.row0 + 16 > n_rows_kv) {
            report_error(kErrIndex);
            t.row0 = 0u;
          }
        }
        return t;
      };
      auto fetch = [&](uint4(&x)[NLD], const uint16_t* base, const TileRef& t) {
#pragma unroll
        for (int i = 0; i < NLD; ++i) {
          const int rr = min(RPI * i + rsub, t.nvalid - 1);
          x[i] = ldg_stream(base + ((int64_t)t.row0 + rr) * D + 8 * u_lane);
        }
      };
      if (first < k1) {
        uint4 kr[NLD], vr[NLD];
        TileRef cur = tile_at(first);
        fetch(kr, Kp, cur);
        fetch(vr, Vp, cur);
        for (int k = first; k < k1; k += kRoutedWarps) {
          const int kn = k + kRoutedWarps;
          const bool more = kn < k1;
          TileRef nx = cur;
          if (more) nx = tile_at(kn);
          store_rows<D>(tile, kr, lane);
          if (more) fetch(kr, Kp, nx);
          __syncwarp();
          uint32_t b0, b1;
          qk_softmax<D>(st, tile, cur.nvalid, qfrag, a.scale_log2, lane, b0, b1);
          __syncwarp();
          store_rows<D>(tile, vr, lane);
          if (more) fetch(vr, Vp, nx);
          __syncwarp();
          pv<D>(st, tile, b0, b1, lane);
          __syncwarp();
          cur = nx;
        }
      }

      // warp partials -> shared memory
      __syncthreads();  // every warp is done with its tile before red_o reuses the region
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
      // CTA combine over warps: whole unit -> output; shared unit -> partial slot c + unit
      float* slot = sp.part + (int64_t)(c + unit) * kPartFloats;
      if (!whole) wait_route();  // the merge count is cleared by the route kernel
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
        if (whole) {
          const int64_t head = (int64_t)b * a.hq + (int64_t)h * a.R + n;
          a.out[head * D + dd] = den > 0.f ? acc / den : 0.f;
          if (dd == 0 && a.lse != nullptr)
            a.lse[head] = den > 0.f ? (M + __log2f(den)) * 0.69314718055994530942f : -INFINITY;
        } else {
          slot[n * D + dd] = acc;
          if (dd == 0) {
            slot[kMaxHeadsPerKv * D + n] = M;
            slot[kMaxHeadsPerKv * D + kMaxHeadsPerKv + n] = den;
          }
        }
      }
      if (whole) continue;
      // publish the partial, count it; the last of the unit's CTAs merges
      __threadfence();
      __syncthreads();
      const int cfirst = slice_of(U0, T, Ge), clast = slice_of(U1 - 1, T, Ge);
      if (tid == 0) {
        const int done = atomicAdd(sp.count + unit, 1);
        misc[0] = done == clast - cfirst;
      }
      __syncthreads();
      if (!misc[0]) continue;
      __threadfence();
      // merge the unit's nc partials: running maxima and denominators to shared
      // memory (red_o is free again), per-head weights, then every output
      // element as one unrolled pass over the partial numerators
      const int nc = clast - cfirst + 1;
      float* wm = red_o;                           // [nc][8] maxima, then weights
      float* wl = red_o + nc * kMaxHeadsPerKv;     // [nc][8] denominators
      for (int i = tid; i < nc * a.R; i += kRoutedThreads) {
        const int cc = i / a.R, n = i - cc * a.R;
        const float* ps = sp.part + (int64_t)(cfirst + cc + unit) * kPartFloats + kMaxHeadsPerKv * D;
        wm[cc * kMaxHeadsPerKv + n] = __ldcg(ps + n);
        wl[cc * kMaxHeadsPerKv + n] = __ldcg(ps + kMaxHeadsPerKv + n);
      }
      __syncthreads();
      if (tid < a.R) {
        const int n = tid;
        float M = -INFINITY;
        for (int cc = 0; cc < nc; ++cc) M = fmaxf(M, wm[cc * kMaxHeadsPerKv + n]);
        float den = 0.f;
        for (int cc = 0; cc < nc; ++cc) {
          const float f = M == -INFINITY ? 0.f : ex2(wm[cc * kMaxHeadsPerKv + n] - M);  // -inf -> 0
          wm[cc * kMaxHeadsPerKv + n] = f;
          den = fmaf(wl[cc * kMaxHeadsPerKv + n], f, den);
        }
        misc[8 + n] = __float_as_int(M);
        misc[16 + n] = __float_as_int(den);
      }
      __syncthreads();
      for (int i = tid; i < a.R * D; i += kRoutedThreads) {
        const int n = i / D, dd = i - n * D;
        const float* po = sp.part + (int64_t)(cfirst + unit) * kPartFloats + n * D + dd;
        float acc = 0.f;
#pragma unroll 8
        for (int cc = 0; cc < nc; ++cc) acc = fmaf(__ldcg(po + (int64_t)cc * kPartFloats), wm[cc * kMaxHeadsPerKv + n], acc);
        const float M = __int_as_float(misc[8 + n]), den = __int_as_float(misc[16 + n]);
        const int64_t head = (int64_t)b * a.hq + (int64_t)h * a.R + n;
        a.out[head * D + dd] = den > 0.f ? acc / den : 0.f;
        if (dd == 0 && a.lse != nullptr)
          a.lse[head] = den > 0.f ? (M + __log2f(den)) * 0.69314718055994530942f : -INFINITY;
      }
    }
  }
  wait_route();  // no CTA leaves before the route kernel's writes are complete
}

}  // namespace hga
