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
//   R1  chunk scores: each CTA scores 1/P of the candidate chunks 1..nf-2 with
//       the head-summed query (sum_i q_i . s_c = (sum_i q_i) . s_c) and writes
//       the 64-bit keys (score, then lower id) into every CTA's shared memory.
//   --  cluster barrier
//   R2  every CTA sorts all keys (bitonic, shared memory) and takes the top k;
//       kept chunk ids are put in ascending order.
//   R3  group scores: each CTA scores the groups of 1/P of the kept chunks and
//       broadcasts a bit mask of the top-G groups per chunk.
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

constexpr int kRoutedWarps = 4;
constexpr int kRoutedThreads = kRoutedWarps * 32;

struct RoutedArgs {
  KvView kv;
  SumView sv;
  const uint16_t* q;  // [B][Hq][D]
  int hq, R;
  int C, g, k, G;     // routing parameters (G already <= C/g)
  int n_pad;          // power of two >= max candidates (max_chunks - 2), >= 2
  int kcap;           // >= kept chunks for any length (min(k, max_chunks - 2)), >= 1
  float scale_log2;   // softmax scale * log2(e)
  float* out;         // [B][Hq][D]
  float* lse;         // [B][Hq] or null
  int32_t* idx_out;   // [B][Hkv][idx_stride] or null
  int32_t* n_idx_out; // [B][Hkv] or null
  const int32_t* idx_in;
  const int32_t* n_idx_in;
  int idx_stride;
};

// Shared-memory carve-up (byte offsets), identical on host and device.
struct RoutedSmem {
  int qsum, keys, sel_tmp, sel, gmask, gstart, gsc, rows, red_o, red_m, red_l, cta_o, cta_m, cta_l,
      qfrag, total;
  __host__ __device__ static int up16(int x) { return (x + 15) & ~15; }
  __host__ __device__ RoutedSmem(int D, int n_pad, int kcap, int gk) {
    int o = 0;
    qsum = o;    o = up16(o + 4 * D);
    keys = o;    o = up16(o + 8 * n_pad);
    sel_tmp = o; o = up16(o + 4 * kcap);
    sel = o;     o = up16(o + 4 * kcap);
    gmask = o;   o = up16(o + 4 * kcap);
    gstart = o;  o = up16(o + 4 * kcap * gk);
    gsc = o;     o = up16(o + 4 * kRoutedWarps * 32);
    rows = o;    o = up16(o + 4 * kEntryBatch);
    red_o = o;   o = up16(o + 4 * kRoutedWarps * kMaxHeadsPerKv * D);
    red_m = o;   o = up16(o + 4 * kRoutedWarps * kMaxHeadsPerKv);
    red_l = o;   o = up16(o + 4 * kRoutedWarps * kMaxHeadsPerKv);
    cta_o = o;   o = up16(o + 4 * kMaxHeadsPerKv * D);
    cta_m = o;   o = up16(o + 4 * kMaxHeadsPerKv);
    cta_l = o;   o = up16(o + 4 * kMaxHeadsPerKv);
    qfrag = o;   o = up16(o + 16 * 32 * (D / 32));
    total = o;
  }
};

// Block-wide bitonic sort of n (power of two) keys, descending.
__device__ __forceinline__ void bitonic_sort_desc(uint64_t* keys, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t a = keys[lo], b = keys[hi];
        if ((a < b) == desc) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

// Dot product of one bf16 summary row (16 B per lane, LPR lanes) with qsum.
template <int D>
__device__ __forceinline__ float row_dot_partial(const uint4& v, const float* qsum, int col) {
  const float4 a = *reinterpret_cast<const float4*>(qsum + col);
  const float4 c = *reinterpret_cast<const float4*>(qsum + col + 4);
  float s = bf16_lo(v.x) * a.x;
  s = fmaf(bf16_hi(v.x), a.y, s);
  s = fmaf(bf16_lo(v.y), a.z, s);
  s = fmaf(bf16_hi(v.y), a.w, s);
  s = fmaf(bf16_lo(v.z), c.x, s);
  s = fmaf(bf16_hi(v.z), c.y, s);
  s = fmaf(bf16_lo(v.w), c.z, s);
  s = fmaf(bf16_hi(v.w), c.w, s);
  return s;
}

template <int LPR>
__device__ __forceinline__ float reduce_lanes(float s) {
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
  return s;
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
  constexpr int LPR = D / 8, RPI = 32 / LPR;

  const int gk = a.G;
  const RoutedSmem lay(D, a.n_pad, a.kcap, gk);
  float* qsum = reinterpret_cast<float*>(smem + lay.qsum);
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem + lay.keys);
  int* sel_tmp = reinterpret_cast<int*>(smem + lay.sel_tmp);
  int* sel = reinterpret_cast<int*>(smem + lay.sel);
  uint32_t* gmask = reinterpret_cast<uint32_t*>(smem + lay.gmask);
  int* gstart = reinterpret_cast<int*>(smem + lay.gstart);
  float* gsc = reinterpret_cast<float*>(smem + lay.gsc);
  uint32_t* rows = reinterpret_cast<uint32_t*>(smem + lay.rows);
  float* red_o = reinterpret_cast<float*>(smem + lay.red_o);
  float* red_m = reinterpret_cast<float*>(smem + lay.red_m);
  float* red_l = reinterpret_cast<float*>(smem + lay.red_l);
  float* cta_o = reinterpret_cast<float*>(smem + lay.cta_o);
  float* cta_m = reinterpret_cast<float*>(smem + lay.cta_m);
  float* cta_l = reinterpret_cast<float*>(smem + lay.cta_l);
  uint4* qfrag = reinterpret_cast<uint4*>(smem + lay.qfrag);

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

  if (kRouting) {
    // Peers write into this CTA's shared memory in R1; every CTA of the cluster
    // must have started first. Arrive now, wait just before the first remote store.
    cluster_arrive_relaxed();
    for (int e = tid; e < D; e += kRoutedThreads) {
      float s = 0.f;
      for (int i = 0; i < a.R; ++i) s += bf16_to_f(qb[(int64_t)i * D + e]);
      qsum[e] = s;
    }
    for (int i = n_cand + tid; i < a.n_pad; i += kRoutedThreads) keys[i] = 0ull;
    __syncthreads();

    cluster_wait();

    // R1: score this CTA's share of the candidates; broadcast keys to the cluster.
    const bool sort_needed = n_cand > r;
    if (sort_needed) {
      const int c0 = (int)((int64_t)n_cand * cr / P), c1 = (int)((int64_t)n_cand * (cr + 1) / P);
      const int nsg = kRoutedWarps * RPI;
      const int sg = warp * RPI + lane / LPR;
      const int col = (lane % LPR) * 8;
      for (int base = c0; base < c1; base += 4 * nsg) {
        uint4 v[4];
        int cand[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          cand[u] = base + sg + u * nsg;
          v[u] = make_uint4(0, 0, 0, 0);
          if (cand[u] < c1) {
            const int c = cand[u] + 1;
            int page = 0;
            bool ok = true;
            if (paged) {
              page = __ldg(a.kv.page_table + (int64_t)b * a.kv.max_pages + c);
              ok = (unsigned)page < (unsigned)a.kv.num_pages;
              if (!ok && (lane % LPR) == 0) report_error(kErrPage);
            }
            if (ok) v[u] = ldg_nc(a.sv.chunk + a.sv.chunk_off(paged, b, h, hkv, c, page) + col);
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float s = reduce_lanes<LPR>(row_dot_partial<D>(v[u], qsum, col));
          if (cand[u] < c1 && (lane % LPR) == 0) {
            const uint64_t key = route_key(s, (uint32_t)(cand[u] + 1));
            for (int pr = 0; pr < P; ++pr) cluster.map_shared_rank(keys, pr)[cand[u]] = key;
          }
        }
      }
    }
    cluster.sync();

    // R2: top-r chunks, ascending ids.
    if (sort_needed) {
      bitonic_sort_desc(keys, a.n_pad);
      for (int i = tid; i < r; i += kRoutedThreads) sel_tmp[i] = (int)route_key_id(keys[i]);
      __syncthreads();
      for (int i = tid; i < r; i += kRoutedThreads) {
        const int c = sel_tmp[i];
        int rank = 0;
        for (int j = 0; j < r; ++j) rank += sel_tmp[j] < c;
        sel[rank] = c;
      }
    } else {
      for (int i = tid; i < r; i += kRoutedThreads) sel[i] = i + 1;
    }
    __syncthreads();

    // R3: group top-G inside this CTA's share of the kept chunks.
    const bool all_groups = gk >= gpc;
    if (!all_groups) {
      const int s0 = (int)((int64_t)r * cr / P), s1 = (int)((int64_t)r * (cr + 1) / P);
      const int sub = lane / LPR, col = (lane % LPR) * 8;
      for (int i = s0 + warp; i < s1; i += kRoutedWarps) {
        const int c = sel[i];
        int page = 0;
        bool ok = true;
        if (paged) {
          page = __ldg(a.kv.page_table + (int64_t)b * a.kv.max_pages + c);
          ok = (unsigned)page < (unsigned)a.kv.num_pages;
        }
        const uint16_t* gbase = a.sv.group + a.sv.group_off(paged, b, h, hkv, c, page) + col;
        for (int j0 = 0; j0 < gpc; j0 += 4 * RPI) {
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = j0 + sub + u * RPI;
            v[u] = (ok && j < gpc) ? ldg_nc(gbase + (int64_t)j * D) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = j0 + sub + u * RPI;
            const float s = reduce_lanes<LPR>(row_dot_partial<D>(v[u], qsum, col));
            if (j < gpc && (lane % LPR) == 0) gsc[warp * 32 + j] = s;
          }
        }
        __syncwarp();
        bool keep = false;
        if (lane < gpc) {
          const float tj = gsc[warp * 32 + lane];
          int rank = 0;
          for (int l = 0; l < gpc; ++l) {
            const float tl = gsc[warp * 32 + l];
            rank += (tl > tj) || (tl == tj && l < lane);
          }
          keep = rank < gk;
        }
        const uint32_t mask = __ballot_sync(0xFFFFFFFFu, keep);
        if (lane == 0)
          for (int pr = 0; pr < P; ++pr) cluster.map_shared_rank(gmask, pr)[i] = mask;
        __syncwarp();
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
      attend_tiles<D>(st, rows, n_e, warp, kRoutedWarps, Kp, Vp, qfrag, a.scale_log2, lane);
    }

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
    // CTA combine over warps
    for (int i = tid; i < a.R * D; i += kRoutedThreads) {
      const int n = i / D, dd = i - n * D;
      float M = -INFINITY;
      for (int w = 0; w < kRoutedWarps; ++w) M = fmaxf(M, red_m[w * kMaxHeadsPerKv + n]);
      float acc = 0.f, den = 0.f;
      if (M != -INFINITY) {
        for (int w = 0; w < kRoutedWarps; ++w) {
          const float mw = red_m[w * kMaxHeadsPerKv + n];
          if (mw == -INFINITY) continue;
          const float f = ex2(mw - M);
          acc = fmaf(red_o[(w * kMaxHeadsPerKv + n) * D + dd], f, acc);
          den = fmaf(red_l[w * kMaxHeadsPerKv + n], f, den);
        }
      }
      cta_o[n * D + dd] = acc;
      if (dd == 0) {
        cta_m[n] = M;
        cta_l[n] = den;
      }
    }
    cluster.sync();
    // cluster combine: CTA cr finalises heads cr, cr + P, ...
    for (int n = cr; n < a.R; n += P) {
      for (int dd = tid; dd < D; dd += kRoutedThreads) {
        float M = -INFINITY;
        for (int pr = 0; pr < P; ++pr) M = fmaxf(M, cluster.map_shared_rank(cta_m, pr)[n]);
        float acc = 0.f, den = 0.f;
        if (M != -INFINITY) {
          for (int pr = 0; pr < P; ++pr) {
            const float mp = cluster.map_shared_rank(cta_m, pr)[n];
            if (mp == -INFINITY) continue;
            const float f = ex2(mp - M);
            acc = fmaf(cluster.map_shared_rank(cta_o, pr)[n * D + dd], f, acc);
            den = fmaf(cluster.map_shared_rank(cta_l, pr)[n], f, den);
          }
        }
        const int64_t head = (int64_t)b * a.hq + (int64_t)h * a.R + n;
        a.out[head * D + dd] = den > 0.f ? acc / den : 0.f;
        if (dd == 0 && a.lse != nullptr)
          a.lse[head] = den > 0.f ? (M + __log2f(den)) * 0.69314718055994530942f : -INFINITY;
      }
    }
    cluster.sync();
  }
}

}  // namespace hga
