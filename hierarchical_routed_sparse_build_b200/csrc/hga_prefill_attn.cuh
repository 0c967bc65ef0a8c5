// Chunked-prefill attention on the 5th-generation tensor cores (tcgen05, TMEM).
//
// "Hierarchical Global Attention (HGA)", abstract: exact attention over the
// routed tokens. For prefill, a block of queries at positions P .. P+63 shares
// one routed cache set T (from hga_route_blocks); query p of the block attends
// to T plus the block's own tokens P .. P+p (causal). Per (block, KV head) that
// is a dense contraction: Q [R heads x 64 queries, d] against the routed keys.
//
// One CTA (one warpgroup, 128 threads) per (block, KV head, 128-row M tile); the
// M tile holds two query heads x 64 queries, row = head_in_tile * 64 + p.
// Keys are processed in tiles of 64:
//   S   = Q K^T   tcgen05.mma M128 N64, K = 128 head dims (8 x K16), fp32 in TMEM
//   P   = softmax rows in registers (tcgen05.ld of S; thread = row), bf16 to smem
//   O  += P V     tcgen05.mma M128 N128, K = 64 keys (4 x K16), fp32 in TMEM
// Operands are staged in 128-byte-swizzled shared memory: Q (K-major, two
// 64-column halves), K tiles (K-major B operand of QK^T), V tiles (the same
// bytes read as the MN-major B operand of PV), P (K-major A operand of PV).
// K/V tiles are gathered row by row with cp.async (double-buffered stages), since
// the routed keys are arbitrary runs of rows. One thread issues the MMAs and
// commits them to mbarriers; every wait is bounded and reports kErrTimeout.
//
// Exit after an expired wait: the CTA stops issuing MMAs and copies, then every
// thread waits (bounded) for the last S and the last PV it committed, so that no
// tcgen05.mma is outstanding when tensor memory is released. Only if one of
// those final waits also expires (an MMA that never completes, which no input
// can cause) does the CTA leave without deallocating, rather than free columns
// an MMA may still write; the timeout is reported either way and no output row
// of the CTA is written.
// The softmax keeps a reference maximum per row and rescales the TMEM
// accumulator only when a new maximum exceeds it by more than 2^8 (exact: the
// final division uses the same reference).
#pragma once

#include "hga_common.cuh"
#include "hga_tcgen05.cuh"

namespace hga {

constexpr int kPfRows = 128;    // M tile
constexpr int kPfKeys = 64;     // keys per tile
constexpr int kPfThreads = 128;
constexpr float kRescaleLog2 = 8.0f;

struct PrefillAttnArgs {
  const uint16_t* q;   // [T][Hq][128]
  int hq, R, T, block;  // block == 64
  const uint16_t* k;   // [Hkv][Lmax][128] (batch 1, contiguous)
  const uint16_t* v;
  int hkv, max_len;
  int cache_len;       // query i sits at position cache_len + i
  int growing;         // nonzero: block b's routed tokens lie in [0, cache_len + b * block)
  const int32_t* idx;  // [n_blocks][Hkv][idx_stride] routed cache tokens
  const int32_t* n_idx;
  int idx_stride;
  float scale_log2;
  float* out;          // [T][Hq][128]
  int fail_at_tile;    // test hook: >= 0 makes key tile j's S wait report expiry after it has completed
};

// Dynamic shared memory, offsets from a 1024-byte aligned base.
struct PrefillSmem {
  static constexpr int kQ = 0;                         // 2 halves x [128 rows x 128 B]
  static constexpr int kK = kQ + 2 * 16384;            // 2 stages x 2 halves x [64 x 128 B]
  static constexpr int kV = kK + 2 * 16384;            // 2 stages x 2 halves x [64 x 128 B]
  static constexpr int kP = kV + 2 * 16384;            // [128 rows x 128 B]
  static constexpr int kBar = kP + 16384;              // bar_s, bar_o, tmem slot, abort flag
  static constexpr int kTotal = kBar + 64;
};

__device__ __forceinline__ uint32_t sw128(int row, int unit) {
  return (uint32_t)(row * 128 + ((unit ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(kPfThreads, 2) prefill_attn_kernel(const PrefillAttnArgs a) {
  constexpr int D = 128;
  extern __shared__ __align__(1024) unsigned char pf_smem[];
  unsigned char* smem = pf_smem;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int m_tiles = a.R * a.block / kPfRows;
  const int mt = blockIdx.x % m_tiles;
  const int unit = blockIdx.x / m_tiles;  // block * hkv + h
  const int blk = unit / a.hkv, h = unit % a.hkv;

  uint64_t* bar_s = reinterpret_cast<uint64_t*>(smem + PrefillSmem::kBar);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  if ((smem_u32(smem) & 1023u) != 0u) {  // swizzle atoms need 1024-byte alignment
    if (tid == 0) report_error(kErrIndex);
    return;
  }

  // rows of this tile: r = tid; head = 2*mt + r/64 within the KV group, p = r % 64
  const int r = tid;
  const int head_local = (mt * kPfRows + r) / a.block, p = (mt * kPfRows + r) % a.block;
  const int qi = blk * a.block + p;
  const int64_t q_row = (int64_t)qi * a.hq + (int64_t)h * a.R + head_local;
  const int own0 = a.cache_len + blk * a.block;  // first own token of the block
  const int hist = a.growing ? own0 : a.cache_len;  // routed tokens lie in [0, hist)

  int n_cache = __ldg(a.n_idx + unit);
  if (n_cache < 0 || n_cache > a.idx_stride) {
    if (tid == 0) report_error(kErrIndex);
    n_cache = 0;
  }
  const int n_keys = n_cache + a.block;
  const int n_tiles = (n_keys + kPfKeys - 1) / kPfKeys;
  const int32_t* ilist = a.idx + (int64_t)unit * a.idx_stride;
  const int64_t head_row0 = (int64_t)h * a.max_len;

  // Key entry e -> token, in two steps so that the list is read one tile ahead
  // without waiting for the load: raw_token() only loads (cache entries), and
  // key_row() validates and turns the token into a K/V row when the copies are
  // issued. Padding entries repeat the block's first own token; they are masked.
  auto raw_token = [&](int e) -> int {
    return e < n_cache ? __ldg(ilist + e) : (e < n_keys ? own0 + (e - n_cache) : own0);
  };
  auto key_row = [&](int e, int tok) -> int64_t {
    if (e < n_cache && (tok < 0 || tok >= hist)) {
      report_error(kErrIndex);
      tok = own0;
    }
    return head_row0 + tok;
  };

  // stage Q (row-wise units, 16 per row) and key tile 0
  unsigned char* sQ = smem + PrefillSmem::kQ;
  for (int i = tid; i < kPfRows * 16; i += kPfThreads) {
    const int rr = i >> 4, u = i & 15;
    const int hl = (mt * kPfRows + rr) / a.block, pp = (mt * kPfRows + rr) % a.block;
    const int64_t row = (int64_t)(blk * a.block + pp) * a.hq + (int64_t)h * a.R + hl;
    cp_async16(sQ + (u >> 3) * 16384 + sw128(rr, u & 7), a.q + row * D + 8 * u);
  }
  // Thread tid copies unit (tid % 16) of keys tid/16 + 8i (i < 8) of a tile: 16
  // consecutive threads cover one 256-byte row. All eight row lookups are
  // issued before the first copy (the copies are ordered memory operations).
  const int cu = tid & 15, ck = tid >> 4;
  auto tile_tokens = [&](int j, int (&tok)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) tok[i] = raw_token(j * kPfKeys + ck + 8 * i);
  };
  auto issue_tile = [&](int j, const int (&tok)[8], int st) {
    unsigned char* sK = smem + PrefillSmem::kK + st * 16384;
    unsigned char* sV = smem + PrefillSmem::kV + st * 16384;
    int64_t rows[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) rows[i] = key_row(j * kPfKeys + ck + 8 * i, tok[i]);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t off = (cu >> 3) * 8192 + sw128(ck + 8 * i, cu & 7);
      cp_async16(sK + off, a.k + rows[i] * D + 8 * cu);
      cp_async16(sV + off, a.v + rows[i] * D + 8 * cu);
    }
  };
  int next_tok[8];
  tile_tokens(0, next_tok);
  issue_tile(0, next_tok, 0);
  cp_async_commit();
  if (n_tiles > 1) tile_tokens(1, next_tok);

  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 64;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  constexpr uint32_t kIdescS = umma_idesc_bf16_f32(kPfRows, kPfKeys, false);
  constexpr uint32_t kIdescO = umma_idesc_bf16_f32(kPfRows, D, true);
  const uint32_t aQ = smem_u32(sQ), aP = smem_u32(smem + PrefillSmem::kP);

  float m_ref = -INFINITY, l_sum = 0.f;
  const float sl = a.scale_log2;
  bool ok = true;
  // index of the last S and PV committed (every thread follows the same control
  // flow, so all agree); the exit waits for both before releasing tensor memory
  int last_s = -1, last_o = -1;

  for (int j = 0; j < n_tiles; ++j) {
    const int st = j & 1;
    cp_async_wait<0>();
    fence_async_smem();
    __syncthreads();
    if (*abort_flag) break;
    // S = Q K_j^T
    last_s = j;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t aK = smem_u32(smem + PrefillSmem::kK + st * 16384);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t da = umma_desc_sw128(aQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        const uint64_t db = umma_desc_sw128(aK + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
        umma_bf16(tS, da, db, kIdescS, kk > 0);
      }
      umma_commit(bar_s);
    }
    // stage j-1 is free once PV_{j-1} has completed; then prefetch tile j+1 into it
    if (j >= 1 && !mbar_wait_bounded(bar_o, (uint32_t)((j - 1) & 1))) ok = false;
    if (j + 1 < n_tiles && ok) issue_tile(j + 1, next_tok, st ^ 1);
    cp_async_commit();
    if (j + 2 < n_tiles) tile_tokens(j + 2, next_tok);  // list entries of the tile after next
    if (!mbar_wait_bounded(bar_s, (uint32_t)(j & 1)) || j == a.fail_at_tile) ok = false;
    tc_fence_after();

    // softmax of this thread's row; only tiles reaching past the routed cache
    // entries need a mask (the block's own tokens are causal, the rest is padding)
    uint32_t sv[2][32];
    tmem_ld32(tS + lane_off + 0, sv[0]);
    tmem_ld32(tS + lane_off + 32, sv[1]);
    tmem_wait_ld();
    // key entry e is attended by this row iff it is a cache entry or an own token
    // at or before the row's query: e < n_cache + p + 1 (and e < n_keys)
    const int lim = min(n_cache + p + 1, n_keys) - j * kPfKeys;  // columns c < lim
    if (lim < kPfKeys) {
#pragma unroll
      for (int c = 0; c < kPfKeys; ++c)
        if (c >= lim) sv[c >> 5][c & 31] = __float_as_uint(-INFINITY);
    }
    float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      mx0 = fmaxf(mx0, __uint_as_float(sv[0][c]));
      mx1 = fmaxf(mx1, __uint_as_float(sv[0][c + 1]));
      mx2 = fmaxf(mx2, __uint_as_float(sv[1][c]));
      mx3 = fmaxf(mx3, __uint_as_float(sv[1][c + 1]));
    }
    const float tmax = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl;  // sl > 0
    const bool need = tmax > m_ref + kRescaleLog2 || (m_ref == -INFINITY && tmax != -INFINITY);
    float alpha = 1.f;
    if (need) {
      alpha = m_ref == -INFINITY ? 0.f : ex2(m_ref - tmax);
      m_ref = tmax;
      l_sum *= alpha;
    }
    // (warp-uniform condition; skipped once a wait has expired, as PV_{j-1} may
    // then still be writing the accumulator)
    if (j >= 1 && __any_sync(0xFFFFFFFFu, need && alpha != 1.f) && __all_sync(0xFFFFFFFFu, ok)) {
      // rescale this warp's accumulator rows (PV_{j-1} has completed)
#pragma unroll
      for (int cb = 0; cb < D; cb += 32) {
        uint32_t ov[32];
        tmem_ld32(tO + lane_off + cb, ov);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
        tmem_st32(tO + lane_off + cb, ov);
      }
      tmem_wait_st();
    }
    const float nbase = m_ref == -INFINITY ? 0.f : -m_ref;
    unsigned char* sP = smem + PrefillSmem::kP;
    float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float pv[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) pv[c] = ex2(fmaf(__uint_as_float(sv[u >> 2][8 * (u & 3) + c]), sl, nbase));
      ls0 += pv[0] + pv[4];
      ls1 += pv[1] + pv[5];
      ls2 += pv[2] + pv[6];
      ls3 += pv[3] + pv[7];
      uint4 w;
      w.x = pack_bf16x2(pv[0], pv[1]);
      w.y = pack_bf16x2(pv[2], pv[3]);
      w.z = pack_bf16x2(pv[4], pv[5]);
      w.w = pack_bf16x2(pv[6], pv[7]);
      *reinterpret_cast<uint4*>(sP + sw128(r, u)) = w;
    }
    l_sum += (ls0 + ls1) + (ls2 + ls3);
    if (!ok) *abort_flag = 1;
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) break;
    // O += P V_j
    last_o = j;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t aV = smem_u32(smem + PrefillSmem::kV + st * 16384);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = umma_desc_sw128(aP + kk * 32, 16, 1024);
        const uint64_t db = umma_desc_sw128(aV + kk * 2048, 8192, 1024);
        umma_bf16(tO, da, db, kIdescO, j > 0 || kk > 0);
      }
      umma_commit(bar_o);
    }
  }
  cp_async_wait<0>();
  // drain: the phase of the last committed S and PV must have completed (a
  // phase already seen completes the wait at once)
  bool drained = true;
  if (last_s >= 0 && !mbar_wait_bounded(bar_s, (uint32_t)(last_s & 1))) drained = false;
  if (last_o >= 0 && !mbar_wait_bounded(bar_o, (uint32_t)(last_o & 1))) drained = false;
  tc_fence_after();
  const bool failed = __syncthreads_or(!ok || !drained || *abort_flag || last_o != n_tiles - 1);
  const bool all_drained = !__syncthreads_or(!drained);
  if (failed) {
    if (tid == 0) report_error(kErrTimeout);
  } else {
    const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
    float* orow = a.out + q_row * D;
#pragma unroll
    for (int cb = 0; cb < D; cb += 32) {
      uint32_t ov[32];
      tmem_ld32(tO + lane_off + cb, ov);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; c += 4)
        *reinterpret_cast<float4*>(orow + cb + c) =
            make_float4(__uint_as_float(ov[c]) * inv, __uint_as_float(ov[c + 1]) * inv,
                        __uint_as_float(ov[c + 2]) * inv, __uint_as_float(ov[c + 3]) * inv);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && all_drained) tmem_dealloc(tmem, 256);
}

}  // namespace hga
