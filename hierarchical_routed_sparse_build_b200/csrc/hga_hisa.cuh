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
//   R2  top-m chunks (bucket select, ascending ids), in every CTA
//   T1  the candidate tokens, [0, C) + the kept chunks' tokens + [(nf-1)C, L)
//       (every token when nf <= 2), are split over the CTAs and scored the
//       same way in 16-row batches of K; their 64-bit keys (score bits, then
//       lower position) go to every CTA
//   --  cluster barrier (skipped, with T1 and T2, when the candidates are no
//       more than the tokens to keep)
//   T2  top k_tok tokens (bucket select, ascending positions), in every CTA
//   A   exact attention over the kept tokens: 16-token tiles split over the
//       CTAs and round-robin over the warps (hga_attention.cuh), rows staged
//       in batches of kEntryBatch entries
//   --  warp -> CTA -> cluster softmax combine (finish_attention)
#pragma once

#include "hga_decode.cuh"

namespace hga {

// Shared-memory carve-up (byte offsets), identical on host and device. The
// union region holds the chunk keys, the token keys and the select scratch,
// then the per-warp attention tiles, then the per-warp partial outputs.
struct HisaSmem {
  int qsum, sel, pages, red_m, red_l, cta_o, cta_m, cta_l, qfrag, hist, misc, rows, tsel, uni, ckeys, tkeys,
      scratch, tiles, red_o, total;
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
    hist = o;    o = up16(o + 4 * kBuckets);
    misc = o;    o = up16(o + 4 * 32);
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
      for (int k = 0; k < NLD; ++k) v[k] = dot8(x[k], qv);
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
    select_top_chunks(ckeys, n_cand, r, sel, hist, misc, scratch, kDecodeScratchKeys);
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
    const int e0 = (int)((int64_t)n_ct * cr / P), e1 = (int)((int64_t)n_ct * (cr + 1) / P);
    const int n_rows = e1 - e0;
    const int nb = (n_rows + 15) / 16;
    float qv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) qv[j] = qsum[8 * u + j];
    auto issue = [&](int bi, uint4(&x)[NLD]) {
#pragma unroll
      for (int k = 0; k < NLD; ++k) {
        const int i = min(16 * bi + RPI * k + rsub, n_rows - 1);
        x[k] = ldg_stream(a.kv.k + (int64_t)tok_row(cand_tok(e0 + i)) * D + 8 * u);
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
        const int e = e0 + i;
        const uint64_t key = route_key(score, (uint32_t)cand_tok(e));
        for (int pr = 0; pr < P; ++pr) cluster.map_shared_rank(tkeys, pr)[e] = key;
      }
    };
    uint4 xa[NLD], xb[NLD];
    if (warp < nb) issue(warp, xa);
    if (warp + kRoutedWarps < nb) issue(warp + kRoutedWarps, xb);
    for (int bi = warp; bi < nb; bi += 2 * kRoutedWarps) {
      consume(bi, xa);
      if (bi + 2 * kRoutedWarps < nb) issue(bi + 2 * kRoutedWarps, xa);
      if (bi + kRoutedWarps < nb) {
        consume(bi + kRoutedWarps, xb);
        if (bi + 3 * kRoutedWarps < nb) issue(bi + 3 * kRoutedWarps, xb);
      }
    }
    cluster.sync();
    // top k_tok of the n_ct keys; candidates are in ascending position, so the
    // ordered compaction writes the kept positions ascending
    select_top_chunks(tkeys, n_ct, k_tok, tsel, hist, misc, scratch, kDecodeScratchKeys);
    __syncthreads();
  }
  const int S = keep_all ? n_ct : k_tok;
  auto entry_tok = [&](int e) -> int { return keep_all ? cand_tok(e) : tsel[e]; };

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
    attend_tiles<D>(st, rows, n_e, warp, kRoutedWarps, a.kv.k, a.kv.v, qfrag, tile, a.scale_log2, lane);
  }
  finish_attention<D>(st, a, cluster, P, cr, b, h, red_o, red_m, red_l, cta_o, cta_m, cta_l);
}

}  // namespace hga
