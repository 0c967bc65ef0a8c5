// Device helpers shared by the routed-attention kernels (sm_100a).
//
// bfloat16 tensors travel as raw uint16 patterns. The gather-heavy decode path
// moves K/V straight from HBM into the registers that feed warp-level bf16
// tensor-core MMAs (mma.sync m16n8k16, fp32 accumulate); see hga_attention.cuh
// for the fragment layouts.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hga {

// ---------------------------------------------------------------- limits

constexpr int kMaxChunks = 4096;       // full chunks per sequence
constexpr int kMaxGroupsPerChunk = 32; // chunk / group
constexpr int kMaxHeadsPerKv = 8;      // query heads sharing one KV head (MMA N = 8)
constexpr int kEntryBatch = 1024;      // routed entries staged per CTA batch
constexpr uint32_t kInvalidRow = 0xFFFFFFFFu;

// ---------------------------------------------------------------- errors

enum DeviceErrorBits : int {
  kErrSeqLen = 1,   // seq_lens[b] outside [0, max_len]
  kErrPage = 2,     // page-table entry outside [0, num_pages)
  kErrIndex = 4,    // routed token outside [0, seq_len), or n_idx > idx_stride
  kErrTimeout = 8,  // a bounded wait ran out
};

// One error word per device (the library's only device state besides code).
__device__ int g_device_error = 0;

__device__ __forceinline__ void report_error(int bits) { atomicOr(&g_device_error, bits); }

// ---------------------------------------------------------------- bf16

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// ---------------------------------------------------------------- PTX wrappers

// 16-byte streaming load: read-only path, no L1 allocation (each K/V byte of the
// routed set is used by exactly one warp once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ldg_nc(const void* p) {
  uint4 r;
  asm("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// 16-byte asynchronous global -> shared copy, cached in L2 only (cp.async.cg).
// Completion is per thread: after cp_async_wait<N>() the issuing thread sees its
// own data, so thread-private staging needs no barrier.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8x8 matrix of 16-bit elements held one row-pair per lane
// (lane l: row l/4, columns 2(l%4), 2(l%4)+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Split cluster barrier (all threads of every CTA of the cluster take part).
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// 2^x on the special-function unit (ex2.approx; -inf -> +0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Order-preserving map of a float to uint32 (larger float -> larger integer);
// -0 is folded onto +0 so that the two compare equal, as in the oracle.
__device__ __forceinline__ uint32_t float_order_bits(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Descending sort key: higher score first, then lower id.
__device__ __forceinline__ uint64_t route_key(float score, uint32_t id) {
  return ((uint64_t)float_order_bits(score) << 32) | (uint64_t)(0xFFFFFFFFu - id);
}
__device__ __forceinline__ uint32_t route_key_id(uint64_t key) {
  return 0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFu);
}

// ---------------------------------------------------------------- views

// The K/V cache as seen by the kernels (see hga_kv in hga.h).
struct KvView {
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* page_table;
  const int32_t* seq_lens;
  int32_t batch, hkv, max_len, page_size, max_pages, num_pages;

  // Row index (in head_dim units) of token t of sequence b, KV head h, or
  // kInvalidRow after reporting a bad page id. t must be in [0, seq_len).
  __device__ __forceinline__ uint32_t row(int b, int h, int t) const {
    if (page_table == nullptr) return (uint32_t)(((int64_t)b * hkv + h) * max_len + t);
    int slot = t / page_size;
    int page = __ldg(page_table + (int64_t)b * max_pages + slot);
    if ((unsigned)page >= (unsigned)num_pages) {
      report_error(kErrPage);
      return kInvalidRow;
    }
    return (uint32_t)(((int64_t)page * hkv + h) * page_size + (t - slot * page_size));
  }

  // Length of sequence b, or 0 after reporting a value outside [0, max_len].
  __device__ __forceinline__ int length(int b) const {
    int L = __ldg(seq_lens + b);
    if (L < 0 || L > max_len) {
      report_error(kErrSeqLen);
      return 0;
    }
    return L;
  }
};

// Summary buffers: contiguous [B][Hkv][max_chunks][...] or paged [page][Hkv][...].
struct SumView {
  uint16_t* chunk;
  uint16_t* group;
  int32_t max_chunks;  // contiguous only
  int32_t gpc;         // groups per chunk
  int32_t d;

  // Offset (elements) of the chunk summary of chunk c of (b, h); for paged
  // caches `page` is the physical page of that chunk.
  __device__ __forceinline__ int64_t chunk_off(bool paged, int b, int h, int hkv, int c, int page) const {
    return paged ? ((int64_t)page * hkv + h) * d : (((int64_t)b * hkv + h) * max_chunks + c) * d;
  }
  __device__ __forceinline__ int64_t group_off(bool paged, int b, int h, int hkv, int c, int page) const {
    return paged ? ((int64_t)page * hkv + h) * gpc * d
                 : ((((int64_t)b * hkv + h) * max_chunks + c) * gpc) * d;
  }
};

}  // namespace hga
