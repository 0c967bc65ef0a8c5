// Chunk and group summaries: one HBM stream over the post-rotary keys.
//
// "Hierarchical Global Attention (HGA)", abstract: routing works on compact
// per-chunk summaries of the rotary-embedded keys, then on per-group summaries
// inside the picked chunks. A summary here is the mean of the keys it covers
// (fp32 accumulation, bfloat16 round-to-nearest store).
//
// One CTA per (chunk, KV head, sequence); warp w reduces groups w, w+8, ...
// Lanes read 16 B each (8 bf16), D/8 lanes per key row, so a warp streams
// 32 * 16 B = 512 contiguous-row bytes per instruction, eight rows of loads in
// flight per lane. Group sums stay in shared memory and are added in group
// order for the chunk mean, so the result does not depend on scheduling.
#pragma once

#include "hga_common.cuh"

namespace hga {

// last_only: the grid has one chunk column and each (head, sequence) CTA
// summarises the chunk that the sequence's last token completed, if it did
// (length a positive multiple of C); used after an append.
template <int D>
__global__ void __launch_bounds__(256) summaries_kernel(KvView kv, SumView sv, int C, int g, int last_only) {
  extern __shared__ float group_acc[];  // [gpc][D]
  const int h = blockIdx.y, b = blockIdx.z;
  const int L = kv.length(b);
  int c = blockIdx.x;
  if (last_only) {
    if (L == 0 || L % C != 0) return;  // uniform over the CTA
    c = L / C - 1;
  }
  if (c >= L / C) return;  // uniform over the CTA
  const bool paged = kv.page_table != nullptr;
  int page = 0;
  int64_t row0;
  if (paged) {
    page = __ldg(kv.page_table + (int64_t)b * kv.max_pages + c);
    if ((unsigned)page >= (unsigned)kv.num_pages) {
      if (threadIdx.x == 0) report_error(kErrPage);
      return;
    }
    row0 = ((int64_t)page * kv.hkv + h) * kv.page_size;
  } else {
    row0 = ((int64_t)b * kv.hkv + h) * kv.max_len + (int64_t)c * C;
  }

  constexpr int LPR = D / 8;    // lanes per key row
  constexpr int RPI = 32 / LPR; // rows per warp instruction
  const int gpc = C / g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int sub = lane / LPR, col = (lane % LPR) * 8;
  const int64_t goff = sv.group_off(paged, b, h, kv.hkv, c, page);
  const float inv_g = 1.0f / (float)g;  // exact when g is a power of two
  const bool g_pow2 = (g & (g - 1)) == 0;

  for (int j = warp; j < gpc; j += nwarps) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    const uint16_t* base = kv.k + (row0 + (int64_t)j * g) * D + col;
    for (int r0 = 0; r0 < g; r0 += 8 * RPI) {
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int r = r0 + sub + i * RPI;
        v[i] = r < g ? ldg_stream(base + (int64_t)r * D) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[0] += bf16_lo(v[i].x); acc[1] += bf16_hi(v[i].x);
        acc[2] += bf16_lo(v[i].y); acc[3] += bf16_hi(v[i].y);
        acc[4] += bf16_lo(v[i].z); acc[5] += bf16_hi(v[i].z);
        acc[6] += bf16_lo(v[i].w); acc[7] += bf16_hi(v[i].w);
      }
    }
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], off);
    if (sub == 0) {
      float m[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        m[i] = g_pow2 ? acc[i] * inv_g : acc[i] / (float)g;
        group_acc[j * D + col + i] = acc[i];
      }
      uint4 o;
      o.x = pack_bf16x2(m[0], m[1]);
      o.y = pack_bf16x2(m[2], m[3]);
      o.z = pack_bf16x2(m[4], m[5]);
      o.w = pack_bf16x2(m[6], m[7]);
      *reinterpret_cast<uint4*>(sv.group + goff + (int64_t)j * D + col) = o;
    }
  }
  __syncthreads();
  const int64_t coff = sv.chunk_off(paged, b, h, kv.hkv, c, page);
  const bool c_pow2 = (C & (C - 1)) == 0;
  const float inv_c = 1.0f / (float)C;
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float s = 0.f;
    for (int j = 0; j < gpc; ++j) s += group_acc[j * D + e];
    float mean = c_pow2 ? s * inv_c : s / (float)C;
    sv.chunk[coff + e] = __bfloat16_as_ushort(__float2bfloat16_rn(mean));
  }
}

// Append one token to every sequence of the cache: K/V rows k_new[b][h],
// v_new[b][h] go to position seq_lens[b] (a contiguous row, or the page slot
// seq_lens[b] / page_size of a paged cache), then seq_lens[b] grows by one.
// One CTA per sequence; the length is read before any thread writes it. A
// length at max_len is reported (kErrSeqLen) and left unchanged.
template <int D>
__global__ void __launch_bounds__(128) append_kernel(KvView kv, uint16_t* k, uint16_t* v, int32_t* seq_lens,
                                                     const uint16_t* k_new, const uint16_t* v_new) {
  const int b = blockIdx.x;
  const int L = seq_lens[b];
  if (L < 0 || L >= kv.max_len) {
    if (threadIdx.x == 0) report_error(kErrSeqLen);
    return;  // uniform over the CTA
  }
  constexpr int U = D / 8;
  for (int i = threadIdx.x; i < kv.hkv * U; i += blockDim.x) {
    const int h = i / U, u = i - h * U;
    const uint32_t row = kv.row(b, h, L);
    if (row == kInvalidRow) continue;  // reported by row()
    const int64_t src = ((int64_t)b * kv.hkv + h) * D + 8 * u;
    *reinterpret_cast<uint4*>(k + (int64_t)row * D + 8 * u) = *reinterpret_cast<const uint4*>(k_new + src);
    *reinterpret_cast<uint4*>(v + (int64_t)row * D + 8 * u) = *reinterpret_cast<const uint4*>(v_new + src);
  }
  __syncthreads();  // every thread has read seq_lens[b]
  if (threadIdx.x == 0) seq_lens[b] = L + 1;
}

}  // namespace hga
