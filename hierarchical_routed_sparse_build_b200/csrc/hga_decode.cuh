// Fused decode (routing + attention in one launch) for group sizes that are a
// whole number of 16-token tiles (g % 16 == 0), one thread-block cluster of P
// CTAs per (sequence, KV head).
//
// "Hierarchical Global Attention (HGA)", abstract: pick chunks by their
// summaries, then the best groups inside the picked chunks, then attend exactly
// over the picked tokens; the first chunk (sink) and the last chunk plus the
// partial tail (local) are always kept (HISA article, two-step block filter).
//
// Compared with routed_kernel's decode mode, group routing is not a separate
// phase: each kept chunk is a job of one warp, which scores that chunk's group
// summaries itself and attends the chosen groups straight away, so the group
// summaries stream in under the K/V gathers and there is no barrier between
// group routing and attention. Phases:
//   R1  chunk scores of this CTA's share of candidates 1..nf-2: every warp
//       streams 16-row batches of summary rows into registers (two batches in
//       flight), dots them with the head-summed query (sum_i q_i) and reduces
//       across lanes with a halving butterfly (one score per lane pair). The
//       64-bit keys (score bits, then lower id) go to every CTA of the cluster.
//   --  cluster barrier
//   R2  every CTA selects the top-k chunk ids (bucket select, ascending ids);
//       warps whose first tile is always kept have its K/V loads in flight.
//   A   the (CTA, warp) slots s = warp * P + cr take kept chunks s, s + P*W, ...
//       and a share of the always-kept tiles (sink chunk, local chunk + tail),
//       the shares balancing the tile counts. A warp first runs its always-kept
//       tiles, then its chunks; for chunk i it waits for the group summaries
//       it fetched with cp.async one chunk earlier, scores them (lanes split
//       each row, shuffle sums), keeps the top-G groups (score desc, index asc)
//       and starts fetching the next chunk's summaries. Every routed tile is
//       16 consecutive tokens of one page, gathered with whole-row 16-byte
//       loads and attended as in hga_attention.cuh, the next tile's K and V in
//       flight during the current tile's math.
//   --  warp -> CTA -> cluster softmax combine (finish_attention).
#pragma once

#include "hga_routed.cuh"

namespace hga {

constexpr int kDecodeScratchKeys = 512;  // boundary-bucket keys ranked in shared memory

// Shared-memory carve-up (byte offsets), identical on host and device. The
// union region holds the routing keys and select scratch, then the per-warp
// attention tiles, then the per-warp partial outputs.
struct DecodeSmem {
  int qsum, sel, pages, red_m, red_l, cta_o, cta_m, cta_l, qfrag, hist, misc, gstage, uni, keys, scratch, tiles,
      red_o, total;
  __host__ __device__ static int up16(int x) { return (x + 15) & ~15; }
  __host__ __device__ DecodeSmem(int D, int n_pad, int kcap, int gpc) {
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
    gstage = o;  o = up16(o + kRoutedWarps * gpc * D * 2);
    uni = o;
    keys = o;
    scratch = up16(keys + 8 * n_pad);
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

// sum over the 8 bf16 of x times q[0..7]
__device__ __forceinline__ float dot8(const uint4 x, const float (&q)[8]) {
  float s0 = bf16_lo(x.x) * q[0];
  float s1 = bf16_hi(x.x) * q[1];
  s0 = fmaf(bf16_lo(x.y), q[2], s0);
  s1 = fmaf(bf16_hi(x.y), q[3], s1);
  s0 = fmaf(bf16_lo(x.z), q[4], s0);
  s1 = fmaf(bf16_hi(x.z), q[5], s1);
  s0 = fmaf(bf16_lo(x.w), q[6], s0);
  s1 = fmaf(bf16_hi(x.w), q[7], s1);
  return s0 + s1;
}

// N partial values per lane, each to be summed over the 2N lanes that share
// bits >= log2(2N) of the lane id. Halving butterfly: at offset o (N, N/2, ...,
// 2) a lane keeps the upper or lower half of its o values and adds the
// partner's matching half; a final xor-1 step completes the sum. Returns the
// total of value index `idx` (same in lanes l and l^1).
template <int N>
__device__ __forceinline__ float butterfly_sum(float (&v)[N], int lane, int& idx) {
  idx = 0;
#pragma unroll
  for (int o = N; o >= 2; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int k = 0; k < o / 2; ++k) {
      const float send = up ? v[k] : v[k + o / 2];
      const float keep = up ? v[k + o / 2] : v[k];
      v[k] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
    if (up) idx += o / 2;
  }
  return v[0] + __shfl_xor_sync(0xFFFFFFFFu, v[0], 1);
}

struct TileRef {
  uint32_t row0;  // row index (head_dim units) of the tile's first token
  int nvalid;     // tokens of the tile inside the context (1..16)
};

template <int D>
__global__ void __launch_bounds__(kRoutedThreads, 2) decode_kernel(const RoutedArgs a) {
  using TG = TileGeom<D>;
  constexpr int U = TG::U, RPI = TG::RPI, NLD = TG::NLD;
  static_assert(NLD == U / 2, "butterfly pairs NLD values over U lanes");
  extern __shared__ __align__(16) unsigned char dec_smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int P = (int)cluster.num_blocks();
  const int cr = (int)cluster.block_rank();
  const int unit = blockIdx.x / P;
  const int hkv = a.kv.hkv;
  const int b = unit / hkv, h = unit % hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = lane % U, rsub = lane / U;

  const int C = a.C, g = a.g, gpc = C / g, gk = a.G;
  const DecodeSmem lay(D, a.n_pad, a.kcap, gpc);
  float* qsum = reinterpret_cast<float*>(dec_smem + lay.qsum);
  int* sel = reinterpret_cast<int*>(dec_smem + lay.sel);
  int* pages = reinterpret_cast<int*>(dec_smem + lay.pages);
  float* red_m = reinterpret_cast<float*>(dec_smem + lay.red_m);
  float* red_l = reinterpret_cast<float*>(dec_smem + lay.red_l);
  float* cta_o = reinterpret_cast<float*>(dec_smem + lay.cta_o);
  float* cta_m = reinterpret_cast<float*>(dec_smem + lay.cta_m);
  float* cta_l = reinterpret_cast<float*>(dec_smem + lay.cta_l);
  uint4* qfrag = reinterpret_cast<uint4*>(dec_smem + lay.qfrag);
  int* hist = reinterpret_cast<int*>(dec_smem + lay.hist);
  int* misc = reinterpret_cast<int*>(dec_smem + lay.misc);
  uint4* gst = reinterpret_cast<uint4*>(dec_smem + lay.gstage) + warp * gpc * U;
  uint64_t* keys = reinterpret_cast<uint64_t*>(dec_smem + lay.keys);
  uint64_t* scratch = reinterpret_cast<uint64_t*>(dec_smem + lay.scratch);
  float* red_o = reinterpret_cast<float*>(dec_smem + lay.red_o);
  uint4* tile = reinterpret_cast<uint4*>(dec_smem + lay.tiles) + warp * TG::kTileSlots;

  const bool paged = a.kv.page_table != nullptr;
  const int L = a.kv.length(b);
  const int nf = L / C;
  const bool dense = nf <= 2;
  const int n_cand = dense ? 0 : nf - 2;
  const int r = n_cand < a.k ? n_cand : a.k;
  const uint16_t* qb = a.q + ((int64_t)b * a.hq + (int64_t)h * a.R) * D;

  // Peers write keys into this CTA's shared memory in R1: every CTA of the
  // cluster must have started first (arrive now, wait before the first store).
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

  // R1 setup; its first loads go out before the head-summed query is formed
  const bool select_needed = n_cand > r;
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
    for (int k = 0; k < NLD; ++k) v[k] = dot8(x[k], qv);
    int idx;
    const float score = butterfly_sum<NLD>(v, lane, idx);
    const int i = 16 * bi + RPI * idx + rsub;
    if ((lane & 1) == 0 && i < n_rows) {
      const int cand = c0 + i;
      const uint64_t key = route_key(score, (uint32_t)(cand + 1));
      for (int pr = 0; pr < P; ++pr) cluster.map_shared_rank(keys, pr)[cand] = key;
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

  // ------------------------------------------------------------------ R1
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
  cluster.sync();

  // ------------------------------------------------------------------- A
  // (set up before the select, which only the routed-chunk tiles depend on)
  const bool all_groups = gk >= gpc;
  const int gsel = all_groups ? gpc : gk;  // groups kept per routed chunk
  const int gt = g / 16;                   // tiles per group
  const int JT = gsel * gt;                // tiles per routed chunk
  const int span = gsel * g;
  const int tail0 = dense ? 0 : (nf - 1) * C;
  const int n_fixed = dense ? (L + 15) / 16 : C / 16 + (L - tail0 + 15) / 16;
  const int S = dense ? L : C + r * span + (L - tail0);
  const int NS = kRoutedWarps * P;
  const int s = warp * P + cr;
  // routed chunk i goes to slot i % NS; this slot's chunks are s, s + NS, ...
  const int n_mine = s < r ? (r - s + NS - 1) / NS : 0;
  // always-kept tiles of this slot: [fa0, fa1) tops up slots that hold one
  // routed chunk fewer (s >= r % NS), the rest [fb0, fb1) is spread evenly
  int fa0 = 0, fa1 = 0, fb0 = 0, fb1 = 0;
  {
    const int rem = r % NS;
    const int n_def = rem == 0 ? 0 : NS - rem;
    const int def_tiles = n_def * JT;
    const bool deficit = rem != 0 && s >= rem;
    if (n_fixed <= def_tiles) {
      if (deficit) {
        fa0 = min(n_fixed, (s - rem) * JT);
        fa1 = min(n_fixed, (s - rem + 1) * JT);
      }
    } else {
      if (deficit) {
        fa0 = (s - rem) * JT;
        fa1 = fa0 + JT;
      }
      const int extra = n_fixed - def_tiles;
      fb0 = def_tiles + (int)((int64_t)extra * s / NS);
      fb1 = def_tiles + (int)((int64_t)extra * (s + 1) / NS);
    }
  }
  const int nA = fa1 - fa0, nF = nA + (fb1 - fb0);
  const int n_tiles = nF + n_mine * JT;

  auto tok_row = [&](int t0) -> uint32_t {
    if (!paged) return (uint32_t)(((int64_t)b * hkv + h) * a.kv.max_len + t0);
    const int slot = t0 / C;  // page = chunk
    return (uint32_t)(((int64_t)pages[slot] * hkv + h) * C + (t0 - slot * C));
  };
  // group summaries of this slot's ci-th routed chunk -> this warp's stage
  auto issue_groups = [&](int ci) {
    const int c = sel[s + ci * NS];
    const uint16_t* src = a.sv.group + a.sv.group_off(paged, b, h, hkv, c, paged ? pages[c] : 0);
    for (int p = lane; p < gpc * U; p += 32) cp_async16(gst + p, src + 8 * p);
    cp_async_commit();
  };
  // top-G groups of the staged chunk (score desc, index asc) as a bit mask
  auto group_mask = [&]() -> uint32_t {
    cp_async_wait<0>();
    __syncwarp();
    int lpr = 32;
    while (lpr * gpc > 32) lpr >>= 1;
    const int row = lane / lpr, part = lane % lpr;
    float v = 0.f;
    if (row < gpc) {
      for (int uu = part; uu < U; uu += lpr) {
        float q8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) q8[j] = qsum[8 * uu + j];
        v += dot8(gst[row * U + uu], q8);
      }
    }
    for (int o = lpr / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    const float mine = __shfl_sync(0xFFFFFFFFu, v, (lane < gpc ? lane : 0) * lpr);
    int rank = 0;
    for (int j = 0; j < gpc; ++j) {
      const float tj = __shfl_sync(0xFFFFFFFFu, v, j * lpr);
      rank += (tj > mine) || (tj == mine && j < lane);
    }
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, lane < gpc && rank < gk);
    __syncwarp();  // every lane has read the stage before it is refilled
    return m;
  };

  int32_t* idx_row = nullptr;
  int idx_cap = 0;
  if (a.idx_out != nullptr) {
    idx_row = a.idx_out + (int64_t)unit * a.idx_stride;
    idx_cap = S;
    if (S > a.idx_stride) {
      if (tid == 0 && cr == 0) report_error(kErrIndex);
      idx_cap = a.idx_stride;
    }
    if (cr == 0 && tid == 0) a.n_idx_out[unit] = S;
  }

  int cur_ci = -1, cur_c = 0;
  uint32_t cur_mask = 0;
  const uint32_t full_mask = gpc >= 32 ? 0xFFFFFFFFu : ((1u << gpc) - 1u);
  // q-th tile of this slot (tiles are asked for in increasing q); also writes
  // the tile's entries of the routed list when one is requested
  auto tile_at = [&](int q) -> TileRef {
    TileRef t;
    int t0, entry0;
    if (q < nF) {
      const int k = q < nA ? fa0 + q : fb0 + (q - nA);
      if (dense || k < C / 16) {
        t0 = 16 * k;
        entry0 = t0;
      } else {
        t0 = tail0 + 16 * (k - C / 16);
        entry0 = C + r * span + (t0 - tail0);
      }
      t.nvalid = min(16, L - t0);
    } else {
      const int kq = q - nF, ci = kq / JT, tt = kq - ci * JT;
      if (ci != cur_ci) {
        cur_ci = ci;
        cur_c = sel[s + ci * NS];
        cur_mask = all_groups ? full_mask : group_mask();
        if (!all_groups && ci + 1 < n_mine) issue_groups(ci + 1);
      }
      const int gr = tt / gt, sub = tt - gr * gt;
      uint32_t m = cur_mask;
      for (int x = 0; x < gr; ++x) m &= m - 1;
      const int j = m ? __ffs(m) - 1 : 0;
      t0 = cur_c * C + j * g + 16 * sub;
      entry0 = C + (s + ci * NS) * span + gr * g + 16 * sub;
      t.nvalid = 16;
    }
    if (idx_row != nullptr && lane < t.nvalid && entry0 + lane < idx_cap) idx_row[entry0 + lane] = t0 + lane;
    t.row0 = tok_row(t0);
    return t;
  };
  auto fetch = [&](uint4(&x)[NLD], const uint16_t* base, const TileRef& t) {
#pragma unroll
    for (int i = 0; i < NLD; ++i) {
      const int rr = min(RPI * i + rsub, t.nvalid - 1);
      x[i] = ldg_stream(base + ((int64_t)t.row0 + rr) * D + 8 * u);
    }
  };

  AttnState<D> st;
  st.init();
  const uint16_t* Kp = a.kv.k;
  const uint16_t* Vp = a.kv.v;
  uint4 kr[NLD], vr[NLD];
  TileRef cur;
  cur.row0 = 0;
  cur.nvalid = 0;
  // a warp whose first tile is always kept loads it under the chunk select
  if (nF > 0) {
    cur = tile_at(0);
    fetch(kr, Kp, cur);
    fetch(vr, Vp, cur);
  }

  // ------------------------------------------------------------------ R2
  if (select_needed) {
    select_top_chunks(keys, n_cand, r, sel, hist, misc, scratch, kDecodeScratchKeys);
  } else {
    for (int i = tid; i < r; i += kRoutedThreads) sel[i] = i + 1;
  }
  __syncthreads();

  if (n_mine > 0 && !all_groups) issue_groups(0);
  if (n_tiles > 0) {
    if (nF == 0) {
      cur = tile_at(0);
      fetch(kr, Kp, cur);
      fetch(vr, Vp, cur);
    }
    for (int q = 0; q < n_tiles; ++q) {
      const bool more = q + 1 < n_tiles;
      TileRef nx = cur;
      if (more) nx = tile_at(q + 1);
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
  finish_attention<D>(st, a, cluster, P, cr, b, h, red_o, red_m, red_l, cta_o, cta_m, cta_l);
}

}  // namespace hga
