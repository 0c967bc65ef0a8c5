// Chunked-prefill attention, warp-specialised: two 128-row Q tiles per CTA
// share every gathered K/V tile, and the softmax of one tile runs while the
// tensor cores work on the other.
//
// "Hierarchical Global Attention (HGA)", abstract: exact attention over the
// routed tokens. As in prefill_attn_kernel, a block of 64 queries shares one
// routed cache set and adds its own tokens causally; the contraction per
// (block, KV head) is Q [R heads x 64 queries, d] against the routed keys.
//
// CTA = (block, KV head, pair of M tiles): tile t in {0, 1} is M tile 2 * mp + t
// (two query heads x 64 queries each). One CTA per SM. Tensor memory (512
// columns) holds, per tile, S/P (64 columns: S of the current 64-key tile in
// fp32, then P as bf16 pairs over its first 32 columns), Q (64 columns, bf16
// pairs, the A operand of S = Q K^T) and O (128 columns, fp32). Shared memory
// holds only a 6-stage ring of gathered K/V tiles (K-major K, the V bytes read
// as the MN-major B operand of O += P V), so the tensor cores read nothing but
// K and V from it.
// Roles:
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1 (thread = row = TMEM lane);
//                    they also load Q into tensor memory and gather the K/V
//                    rows of key tile j+5 with 16-byte cp.async at the end of
//                    iteration j, once the PV products of tile j-1 have freed
//                    its stage (every thread's copies arrive on the stage's
//                    mbarrier when they land)
//   warp 8           tcgen05 issue (one thread) and the TMEM allocation
// The MMA thread staggers the tiles by half a step, S_0(j), PV_1(j-1), S_1(j),
// PV_0(j), so that the tensor cores work on one tile while the other tile's
// softmax runs; S_t(j) waits for PV_t(j-1) (its S/P columns are reused).
// Handshakes (mbarriers; every wait bounded, and a timeout anywhere sets a
// shared abort flag that every other wait checks):
//   kv_full           gatherers -> MMA    stage holds the tile's K and V rows
//   kv_empty          MMA -> gatherers    both PV products of the tile done
//   q_full            softmax -> MMA      Q in tensor memory
//   s_full            MMA -> softmax      S written
//   p_ready           softmax -> MMA      P written (and O rescaled)
//   o_done            MMA -> softmax, MMA PV done: S/P free, O readable
// Masking and the lazy O rescale (threshold 2^8) are those of
// prefill_attn_kernel.
#pragma once

#include "hga_common.cuh"
#include "hga_prefill_attn.cuh"
#include "hga_tcgen05.cuh"

namespace hga {

constexpr int kPf2Stages = 6;
constexpr int kPf2Threads = 288;
constexpr int kPf2Softmax = 256;
constexpr int kPf2MmaWarp = 8;

struct Prefill2Smem {
  static constexpr int kKV = 0;                             // stages x (K 2 x 8 KiB, V 2 x 8 KiB)
  static constexpr int kBar = kKV + kPf2Stages * 32768;
  // mbarrier indices
  static constexpr int bKvFull = 0;                 // [stage], 256 arrivals (cp.async)
  static constexpr int bKvEmpty = bKvFull + kPf2Stages;  // [stage], 1 (commit)
  static constexpr int bSFull = bKvEmpty + kPf2Stages;   // [tile], 1 (commit)
  static constexpr int bPReady = bSFull + 2;        // [tile], 128
  static constexpr int bODone = bPReady + 2;        // [tile], 1 (commit)
  static constexpr int bQFull = bODone + 2;         // 256
  static constexpr int bFinal = bQFull + 1;         // 1 (commit)
  static constexpr int kNumBars = bFinal + 1;
  static constexpr int kSlot = kBar + 8 * kNumBars;  // TMEM base address
  static constexpr int kAbort = kSlot + 4;
  static constexpr int kTotal = kSlot + 16;
};
// tensor-memory columns
constexpr uint32_t kTmS = 0;      // + 64 * tile
constexpr uint32_t kTmQ = 128;    // + 64 * tile
constexpr uint32_t kTmO = 256;    // + 128 * tile
static_assert(Prefill2Smem::kTotal <= 227 * 1024, "shared memory");

__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__global__ void __launch_bounds__(kPf2Threads, 1) prefill_attn2_kernel(const PrefillAttnArgs a) {
  constexpr int D = 128;
  extern __shared__ __align__(1024) unsigned char pf2_smem[];
  unsigned char* smem = pf2_smem;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m_tiles = a.R * a.block / kPfRows;
  const int n_pairs = m_tiles / 2;
  const int mp = blockIdx.x % n_pairs;
  const int unit = blockIdx.x / n_pairs;  // block * hkv + h
  const int blk = unit / a.hkv, h = unit % a.hkv;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Prefill2Smem::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Prefill2Smem::kSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Prefill2Smem::kAbort);
  if ((smem_u32(smem) & 1023u) != 0u) {  // swizzle atoms need 1024-byte alignment
    if (tid == 0) report_error(kErrIndex);
    return;
  }

  int n_cache = __ldg(a.n_idx + unit);
  if (n_cache < 0 || n_cache > a.idx_stride) {
    if (tid == 0) report_error(kErrIndex);
    n_cache = 0;
  }
  const int n_keys = n_cache + a.block;
  const int n_tiles = (n_keys + kPfKeys - 1) / kPfKeys;
  const int own0 = a.cache_len + blk * a.block;  // first own token of the block
  const int hist = a.growing ? own0 : a.cache_len;  // routed tokens lie in [0, hist)

  if (tid == 0) {
    for (int s = 0; s < kPf2Stages; ++s) {
      mbar_init(bars + Prefill2Smem::bKvFull + s, kPf2Softmax);
      mbar_init(bars + Prefill2Smem::bKvEmpty + s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bars + Prefill2Smem::bSFull + t, 1);
      mbar_init(bars + Prefill2Smem::bPReady + t, kPfRows);
      mbar_init(bars + Prefill2Smem::bODone + t, 1);
    }
    mbar_init(bars + Prefill2Smem::bQFull, kPf2Softmax);
    mbar_init(bars + Prefill2Smem::bFinal, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == kPf2MmaWarp) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Bounded wait that gives up early once another thread has set the abort flag.
  auto wait = [&](int bar, uint32_t parity) -> bool {
    for (uint32_t i = 0; i < kMaxSpins; ++i) {
      if (mbar_try_wait(bars + bar, parity)) return true;
      if ((i & 255u) == 255u && *abort_flag) return false;
    }
    *abort_flag = 1;
    report_error(kErrTimeout);
    return false;
  };

  if (warp == kPf2MmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t kIdescS = umma_idesc_bf16_f32(kPfRows, kPfKeys, false);
      constexpr uint32_t kIdescO = umma_idesc_bf16_f32(kPfRows, D, true);
      const uint32_t aKV = smem_u32(smem + Prefill2Smem::kKV);
      bool ok = wait(Prefill2Smem::bQFull, 0);
      if (ok) tc_fence_after();
      // S_t(j) = Q_t K_j^T, once PV_t(j-1) has released the S/P columns
      auto issue_s = [&](int j, int t) -> bool {
        if (j >= 1) {
          if (!wait(Prefill2Smem::bODone + t, (uint32_t)((j - 1) & 1))) return false;
          tc_fence_after();
        }
        const uint32_t aK = aKV + (j % kPf2Stages) * 32768;
        const uint32_t tS = tmem + kTmS + 64 * t, tQ = tmem + kTmQ + 64 * t;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t db = umma_desc_sw128(aK + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
          umma_bf16_tmem_a(tS, tQ + 8 * kk, db, kIdescS, kk > 0);
        }
        umma_commit(bars + Prefill2Smem::bSFull + t);
        return true;
      };
      // O_t += P_t(j) V_j once the softmax threads have written P_t(j)
      auto issue_pv = [&](int j, int t) -> bool {
        if (!wait(Prefill2Smem::bPReady + t, (uint32_t)(j & 1))) return false;
        tc_fence_after();
        const uint32_t aV = aKV + (j % kPf2Stages) * 32768 + 16384;
        const uint32_t tO = tmem + kTmO + 128 * t, tP = tmem + kTmS + 64 * t;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t db = umma_desc_sw128(aV + kk * 2048, 8192, 1024);
          umma_bf16_tmem_a(tO, tP + 8 * kk, db, kIdescO, j > 0 || kk > 0);
        }
        umma_commit(bars + Prefill2Smem::bODone + t);
        if (t == 1) umma_commit(bars + Prefill2Smem::bKvEmpty + j % kPf2Stages);
        return true;
      };
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (!wait(Prefill2Smem::bKvFull + j % kPf2Stages, (uint32_t)((j / kPf2Stages) & 1))) {
          ok = false;
          break;
        }
        fence_async_smem();  // cp.async writes -> tensor-core reads
        tc_fence_after();
        ok = issue_s(j, 0);
        if (ok && j >= 1) ok = issue_pv(j - 1, 1);
        if (ok) ok = issue_s(j, 1);
        if (ok) ok = issue_pv(j, 0);
      }
      if (ok && n_tiles > 0) ok = issue_pv(n_tiles - 1, 1);
      // every MMA of this thread completes before the accumulators are freed
      umma_commit(bars + Prefill2Smem::bFinal);
      mbar_wait_bounded(bars + Prefill2Smem::bFinal, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int t = warp >> 2;                 // Q tile
    const int r = tid & (kPfRows - 1);       // row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int g = (2 * mp + t) * kPfRows + r;
    const int head_local = g / a.block, p = g % a.block;
    const int64_t q_row = (int64_t)(blk * a.block + p) * a.hq + (int64_t)h * a.R + head_local;
    const uint32_t tO = tmem + kTmO + 128 * t;
    const uint32_t tS = tmem + kTmS + 64 * t;
    // this row of Q -> tensor memory (64 columns of bf16 pairs)
    {
      const uint4* qsrc = reinterpret_cast<const uint4*>(a.q + q_row * D);
      uint32_t qw[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = ldg_nc(qsrc + 8 * half + u);
          qw[4 * u] = v.x;
          qw[4 * u + 1] = v.y;
          qw[4 * u + 2] = v.z;
          qw[4 * u + 3] = v.w;
        }
        tmem_st32(tmem + kTmQ + 64 * t + lane_off + 32 * half, qw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars + Prefill2Smem::bQFull);
    }

    // K/V gather: warp w copies rows 8w + 2k + lane/16 (k < 4), unit lane % 16,
    // of K and V; lane (row - 8w) of the warp holds the row's token id, read one
    // tile before it is needed and passed on by shuffles.
    const int32_t* ilist = a.idx + (int64_t)unit * a.idx_stride;
    const int64_t head_row0 = (int64_t)h * a.max_len;
    const int cu = lane & 15, ck = lane >> 4;
    auto raw_token = [&](int e) -> int {
      return e < n_cache ? __ldg(ilist + e) : (e < n_keys ? own0 + (e - n_cache) : own0);
    };
    auto load_token = [&](int jt) -> int { return raw_token(jt * kPfKeys + 8 * warp + (lane & 7)); };
    auto gather = [&](int jt, int tok) {
      unsigned char* stage = smem + Prefill2Smem::kKV + (jt % kPf2Stages) * 32768;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = 8 * warp + 2 * k + ck;
        int tk = __shfl_sync(0xFFFFFFFFu, tok, 2 * k + ck);
        if (jt * kPfKeys + row < n_cache && (tk < 0 || tk >= hist)) {
          report_error(kErrIndex);
          tk = own0;
        }
        const uint32_t off = (cu >> 3) * 8192 + sw128(row, cu & 7);
        cp_async16(stage + off, a.k + (head_row0 + tk) * D + 8 * cu);
        cp_async16(stage + 16384 + off, a.v + (head_row0 + tk) * D + 8 * cu);
      }
      cp_async_mbar_arrive_noinc(bars + Prefill2Smem::bKvFull + jt % kPf2Stages);
    };
    {
      int tk[kPf2Stages - 1];
#pragma unroll
      for (int i = 0; i < kPf2Stages - 1; ++i) tk[i] = load_token(i);
#pragma unroll
      for (int i = 0; i < kPf2Stages - 1; ++i)
        if (i < n_tiles) gather(i, tk[i]);
    }
    int tok_next = load_token(kPf2Stages - 1);  // token of the next tile to gather

    float m_ref = -INFINITY, l_sum = 0.f;
    const float sl = a.scale_log2;
    bool ok = true;
    int o_seen = -1;  // last PV whose completion this thread has waited for
    for (int j = 0; j < n_tiles; ++j) {
      if (!wait(Prefill2Smem::bSFull + t, (uint32_t)(j & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // S is read 32 columns at a time (registers): columns 0-31 for the max,
      // then 32-63 (kept for their exponentials), then 0-31 again.
      const bool masked_tile = (j + 1) * kPfKeys > n_cache;
      auto mask32 = [&](uint32_t (&sv)[32], int c0) {
        if (masked_tile) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int e = j * kPfKeys + c0 + c;
            const bool valid = e < n_cache || (e < n_keys && (e - n_cache) <= p);
            if (!valid) sv[c] = __float_as_uint(-INFINITY);
          }
        }
      };
      auto max32 = [&](const uint32_t (&sv)[32]) -> float {
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          m0 = fmaxf(m0, __uint_as_float(sv[c]));
          m1 = fmaxf(m1, __uint_as_float(sv[c + 1]));
          m2 = fmaxf(m2, __uint_as_float(sv[c + 2]));
          m3 = fmaxf(m3, __uint_as_float(sv[c + 3]));
        }
        return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
      };
      uint32_t sv[32];
      tmem_ld32(tS + lane_off + 0, sv);
      tmem_wait_ld();
      mask32(sv, 0);
      const float mlo = max32(sv);
      tmem_ld32(tS + lane_off + 32, sv);
      tmem_wait_ld();
      mask32(sv, 32);
      const float tmax = fmaxf(mlo, max32(sv)) * sl;  // sl > 0
      const bool need = tmax > m_ref + kRescaleLog2 || (m_ref == -INFINITY && tmax != -INFINITY);
      float alpha = 1.f;
      if (need) {
        alpha = m_ref == -INFINITY ? 0.f : ex2(m_ref - tmax);
        m_ref = tmax;
        l_sum *= alpha;
      }
      if (j >= 1 && __any_sync(0xFFFFFFFFu, need && alpha != 1.f)) {
        // rescale this warp's accumulator rows once PV(j-1) has completed
        if (!wait(Prefill2Smem::bODone + t, (uint32_t)((j - 1) & 1))) {
          ok = false;
          break;
        }
        o_seen = j - 1;
        tc_fence_after();
#pragma unroll 1
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
      float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;
      uint4 pw[8];
      auto exp32 = [&](const uint32_t (&sv)[32], int u0) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float pv[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) pv[c] = ex2(fmaf(__uint_as_float(sv[8 * u + c]), sl, nbase));
          ls0 += pv[0] + pv[4];
          ls1 += pv[1] + pv[5];
          ls2 += pv[2] + pv[6];
          ls3 += pv[3] + pv[7];
          pw[u0 + u].x = pack_bf16x2(pv[0], pv[1]);
          pw[u0 + u].y = pack_bf16x2(pv[2], pv[3]);
          pw[u0 + u].z = pack_bf16x2(pv[4], pv[5]);
          pw[u0 + u].w = pack_bf16x2(pv[6], pv[7]);
        }
      };
      exp32(sv, 4);
      tmem_ld32(tS + lane_off + 0, sv);
      tmem_wait_ld();
      mask32(sv, 0);
      exp32(sv, 0);
      l_sum += (ls0 + ls1) + (ls2 + ls3);
      // P (bf16 pairs, key 2c and 2c+1 in column c) over the first 32 columns of
      // this S buffer, every S value having been read
      uint32_t pc[32];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        pc[4 * u] = pw[u].x;
        pc[4 * u + 1] = pw[u].y;
        pc[4 * u + 2] = pw[u].z;
        pc[4 * u + 3] = pw[u].w;
      }
      tmem_st32(tS + lane_off + 0, pc);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars + Prefill2Smem::bPReady + t);
      // tile j+5 goes into the stage of tile j-1 once both PV products of j-1 are done
      const int jn = j + kPf2Stages - 1;
      if (jn < n_tiles) {
        if (j >= 1 && !wait(Prefill2Smem::bKvEmpty + jn % kPf2Stages, (uint32_t)(((j - 1) / kPf2Stages) & 1))) {
          ok = false;
          break;
        }
        gather(jn, tok_next);
        tok_next = load_token(jn + 1);
      }
    }
    const int jl = n_tiles - 1;
    if (ok && n_tiles > 0 && o_seen < jl && !wait(Prefill2Smem::bODone + t, (uint32_t)(jl & 1))) ok = false;
    tc_fence_after();
    if (ok && !*abort_flag) {
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kPf2MmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace hga
