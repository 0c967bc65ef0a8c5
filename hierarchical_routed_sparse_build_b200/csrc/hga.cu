// libhga: C ABI entry points (include/hga.h) for routed attention on sm_100a.
//
// Host code validates every argument before anything is enqueued, picks the
// launch shape, and launches the kernels of hga_summaries.cuh and
// hga_routed.cuh on the caller's stream. No device memory is allocated here.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <mutex>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "hga.h"
#include "hga_balanced.cuh"
#include "hga_common.cuh"
#include "hga_decode.cuh"
#include "hga_hisa.cuh"
#include "hga_prefill_attn.cuh"
#include "hga_prefill_route.cuh"
#include "hga_routed.cuh"
#include "hga_summaries.cuh"

namespace hga {
namespace {

std::atomic<int> g_ctas_per_head{0};
std::atomic<int> g_decode_kernel{0};  // 0 automatic, 1 phase-by-phase, 2 fused, 3 route + balanced attention
std::atomic<int> g_fail_at_tile{-1};  // test hook of the prefill attention kernel (-1: off)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hga_status check_kv(const hga_kv* kv, bool need_v) {
  if (kv == nullptr || kv->k == nullptr || kv->seq_lens == nullptr) return HGA_ERR_INVALID_ARG;
  if (need_v && kv->v == nullptr) return HGA_ERR_INVALID_ARG;
  if (kv->batch < 1 || kv->n_kv_heads < 1 || kv->max_len < 1 || kv->head_dim < 1)
    return HGA_ERR_INVALID_ARG;
  if (kv->head_dim != 64 && kv->head_dim != 128) return HGA_ERR_UNSUPPORTED;
  if (!aligned16(kv->k) || (need_v && !aligned16(kv->v))) return HGA_ERR_INVALID_ARG;
  if (kv->page_table != nullptr) {
    if (kv->page_size < 1 || kv->max_pages < 1 || kv->num_pages < 1) return HGA_ERR_INVALID_ARG;
    if ((int64_t)kv->max_pages * kv->page_size < kv->max_len) return HGA_ERR_INVALID_ARG;
    if ((int64_t)kv->num_pages * kv->n_kv_heads * kv->page_size >= (int64_t)UINT32_MAX)
      return HGA_ERR_UNSUPPORTED;
  } else {
    if ((int64_t)kv->batch * kv->n_kv_heads * kv->max_len >= (int64_t)UINT32_MAX)
      return HGA_ERR_UNSUPPORTED;
  }
  return HGA_OK;
}

hga_status check_params(const hga_params* p, const hga_kv* kv, bool routing) {
  if (p == nullptr) return HGA_ERR_INVALID_ARG;
  if (!(p->scale >= 0.f) || std::isinf(p->scale)) return HGA_ERR_INVALID_ARG;
  if (!routing) return HGA_OK;
  if (p->chunk < 1 || p->group < 1 || p->chunk % p->group != 0) return HGA_ERR_INVALID_ARG;
  if (p->top_chunks < 1 || p->top_groups < 1 || p->top_groups > p->chunk / p->group)
    return HGA_ERR_INVALID_ARG;
  if (p->chunk / p->group > kMaxGroupsPerChunk) return HGA_ERR_UNSUPPORTED;
  if (kv->max_len / p->chunk > kMaxChunks) return HGA_ERR_UNSUPPORTED;
  if (kv->page_table != nullptr && kv->page_size != p->chunk) return HGA_ERR_UNSUPPORTED;
  return HGA_OK;
}

hga_status check_heads(int32_t n_q_heads, const hga_kv* kv) {
  if (n_q_heads < 1 || n_q_heads % kv->n_kv_heads != 0) return HGA_ERR_INVALID_ARG;
  if (n_q_heads / kv->n_kv_heads > kMaxHeadsPerKv) return HGA_ERR_UNSUPPORTED;
  return HGA_OK;
}

int max_routed(const hga_kv* kv, const hga_params* p) {
  const int C = p->chunk, g = p->group, gk = p->top_groups;
  const int nf_max = kv->max_len / C;
  int best = kv->max_len < 3 * C - 1 ? kv->max_len : 3 * C - 1;  // nf <= 2: dense
  for (int nf = 3; nf <= nf_max; ++nf) {
    const int r = nf - 2 < p->top_chunks ? nf - 2 : p->top_chunks;
    const int tail = kv->max_len - nf * C < C - 1 ? kv->max_len - nf * C : C - 1;
    const int s = 2 * C + r * gk * g + tail;
    if (s > best) best = s;
  }
  return best;
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

int pick_cluster(int units) {
  int P = g_ctas_per_head.load();
  if (P > 0) return P;
  // as many CTAs per (sequence, KV head) as fit in one wave of two CTAs per SM,
  // at most 8 (the portable cluster size)
  P = (2 * sm_count()) / units;
  return P < 1 ? 1 : (P > 8 ? 8 : P);
}

KvView make_kv_view(const hga_kv* kv) {
  KvView v;
  v.k = static_cast<const uint16_t*>(kv->k);
  v.v = static_cast<const uint16_t*>(kv->v);
  v.page_table = kv->page_table;
  v.seq_lens = kv->seq_lens;
  v.batch = kv->batch;
  v.hkv = kv->n_kv_heads;
  v.max_len = kv->max_len;
  v.page_size = kv->page_table ? kv->page_size : 0;
  v.max_pages = kv->page_table ? kv->max_pages : 0;
  v.num_pages = kv->page_table ? kv->num_pages : 0;
  return v;
}

SumView make_sum_view(const hga_kv* kv, const hga_params* p, const void* cs, const void* gs) {
  SumView s;
  s.chunk = const_cast<uint16_t*>(static_cast<const uint16_t*>(cs));
  s.group = const_cast<uint16_t*>(static_cast<const uint16_t*>(gs));
  s.max_chunks = p ? kv->max_len / p->chunk : 0;
  s.gpc = p ? p->chunk / p->group : 1;
  s.d = kv->head_dim;
  return s;
}

float scale_log2(const hga_params* p, int d) {
  const double sc = p->scale > 0.f ? (double)p->scale : 1.0 / std::sqrt((double)d);
  return (float)(sc * 1.4426950408889634074);
}

// Kernel attributes are set once per (kernel, device) and raised only when a
// launch needs more, keeping the per-call host cost to the launch itself.
constexpr int kMaxDevices = 64;

template <int D, int MODE>
cudaError_t configure_routed(int smem_bytes, bool non_portable) {
  static std::atomic<int> smem_set[kMaxDevices];
  static std::atomic<bool> np_set[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  auto kern = routed_kernel<D, MODE>;
  if (smem_bytes > smem_set[dev].load()) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return e;
    smem_set[dev].store(smem_bytes);
  }
  if (non_portable && !np_set[dev].load()) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    np_set[dev].store(true);
  }
  return cudaSuccess;
}

template <int D, int MODE>
cudaError_t launch_routed(const RoutedArgs& a, int units, int P, cudaStream_t stream) {
  const RoutedSmem lay(D, a.n_pad, a.kcap, a.G, a.C / a.g);
  auto kern = routed_kernel<D, MODE>;
  cudaError_t e = configure_routed<D, MODE>(lay.total, P > 8);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3((unsigned)(units * P), 1, 1);
  cfg.blockDim = dim3(kRoutedThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)lay.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

constexpr int kMaxSmemPerCta = 227 * 1024;

template <int MODE>
hga_status run_routed(RoutedArgs a, int D, int units, cudaStream_t stream) {
  if (RoutedSmem(D, a.n_pad, a.kcap, a.G, a.C / a.g).total > kMaxSmemPerCta) return HGA_ERR_UNSUPPORTED;
  const int P = pick_cluster(units);
  cudaError_t e = D == 128 ? launch_routed<128, MODE>(a, units, P, stream)
                           : launch_routed<64, MODE>(a, units, P, stream);
  return e == cudaSuccess ? HGA_OK : HGA_ERR_CUDA;
}

template <int D>
cudaError_t launch_decode(const RoutedArgs& a, int units, int P, cudaStream_t stream) {
  const DecodeSmem lay(D, a.n_pad, a.kcap, a.C / a.g);
  auto kern = decode_kernel<D>;
  static std::atomic<int> smem_set[kMaxDevices];
  static std::atomic<bool> np_set[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (lay.total > smem_set[dev].load()) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
    if (e != cudaSuccess) return e;
    smem_set[dev].store(lay.total);
  }
  if (P > 8 && !np_set[dev].load()) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    np_set[dev].store(true);
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3((unsigned)(units * P), 1, 1);
  cfg.blockDim = dim3(kRoutedThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)lay.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

hga_status run_decode(RoutedArgs a, int D, int units, cudaStream_t stream) {
  if (DecodeSmem(D, a.n_pad, a.kcap, a.C / a.g).total > kMaxSmemPerCta) return HGA_ERR_UNSUPPORTED;
  const int P = pick_cluster(units);
  cudaError_t e = D == 128 ? launch_decode<128>(a, units, P, stream) : launch_decode<64>(a, units, P, stream);
  return e == cudaSuccess ? HGA_OK : HGA_ERR_CUDA;
}

// ---------------------------------------------------------------- balanced decode

// Most tiles one unit can have at any length up to max_len (UnitTiles over L).
int max_unit_tiles(const hga_kv* kv, const hga_params* p) {
  int best = 0;
  const int C = p->chunk;
  // the count depends on L only through nf (capped at top_chunks + 2) and the tail
  for (int L = kv->max_len; L >= 0 && L > kv->max_len - 2 * C; --L) {
    const int t = UnitTiles(L, C, p->group, p->top_chunks, p->top_groups).total();
    if (t > best) best = t;
  }
  const int small = UnitTiles(3 * C - 1 < kv->max_len ? 3 * C - 1 : kv->max_len, C, p->group, p->top_chunks,
                              p->top_groups).total();
  return best > small ? best : small;
}

// Routed tiles of one unit at most (the route kernel's list length).
int max_routed_tiles(const hga_kv* kv, const hga_params* p) {
  const int nf_max = kv->max_len / p->chunk;
  const int cand = nf_max > 2 ? nf_max - 2 : 0;
  const int r = cand < p->top_chunks ? cand : p->top_chunks;
  return r * p->top_groups * (p->group / 16);
}

bool split_applies(const hga_kv* kv, const hga_params* p) {
  return p->group % 16 == 0 && kv->batch <= kSplitMaxBatch;
}

// Workspace of the balanced decode, 256-byte aligned parts: tile lists, partial
// states (one slot per CTA + unit), merge counts.
struct SplitLayout {
  size_t tiles, part, count, total;
  int tile_stride, grid_max;
  SplitLayout(const hga_kv* kv, const hga_params* p, int sms) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t units = (size_t)kv->batch * kv->n_kv_heads;
    tile_stride = max_routed_tiles(kv, p);
    if (tile_stride < 1) tile_stride = 1;
    grid_max = 2 * sms;
    tiles = 0;
    part = up(tiles + units * (size_t)tile_stride * 4);
    count = up(part + ((size_t)grid_max + units) * kPartFloats * 4);
    total = up(count + units * 4);
  }
};

int split_grid(const hga_kv* kv, const hga_params* p, int sms) {
  // at least ~8 tiles per CTA, so that small problems do not spread over more
  // CTAs (and partial merges) than they have work for
  const int64_t t_max = (int64_t)kv->batch * kv->n_kv_heads * max_unit_tiles(kv, p);
  int64_t gsz = t_max / 8;
  if (gsz > 2 * sms) gsz = 2 * sms;
  return gsz < 1 ? 1 : (int)gsz;
}

template <int D>
cudaError_t launch_split(const RoutedArgs& a, const SplitArgs& sp, int units, int P, cudaStream_t stream) {
  const RouteTilesSmem lay1(D, a.n_pad, a.kcap, a.C / a.g);
  const BalancedSmem lay2(D, a.kv.batch, sp.grid);
  auto k1 = route_tiles_kernel<D>;
  auto k2 = balanced_attend_kernel<D>;
  static std::atomic<int> smem1[kMaxDevices], smem2[kMaxDevices];
  static std::atomic<bool> np_set[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (lay1.total > smem1[dev].load()) {
    if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, lay1.total)) != cudaSuccess)
      return e;
    smem1[dev].store(lay1.total);
  }
  if (lay2.total > smem2[dev].load()) {
    if ((e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, lay2.total)) != cudaSuccess)
      return e;
    smem2[dev].store(lay2.total);
  }
  if (P > 8 && !np_set[dev].load()) {
    if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess) return e;
    np_set[dev].store(true);
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3((unsigned)(units * P), 1, 1);
  cfg.blockDim = dim3(kRoutedThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)lay1.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if ((e = cudaLaunchKernelEx(&cfg, k1, a, sp)) != cudaSuccess) return e;
  // the attention kernel is a programmatic dependent of the route kernel: it may
  // start in free SM slots and attend sink / local tiles before the routes exist
  cudaLaunchConfig_t cfg2;
  std::memset(&cfg2, 0, sizeof cfg2);
  cfg2.gridDim = dim3((unsigned)sp.grid, 1, 1);
  cfg2.blockDim = dim3(kRoutedThreads, 1, 1);
  cfg2.dynamicSmemBytes = (size_t)lay2.total;
  cfg2.stream = stream;
  cudaLaunchAttribute attr2[1];
  attr2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr2[0].val.programmaticStreamSerializationAllowed = 1;
  cfg2.attrs = attr2;
  cfg2.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg2, k2, a, sp);
}

hga_status run_split(const RoutedArgs& a, const hga_kv* kv, const hga_params* p, void* workspace, int D,
                     cudaStream_t stream) {
  if (RouteTilesSmem(D, a.n_pad, a.kcap, a.C / a.g).total > kMaxSmemPerCta ||
      BalancedSmem(D, kv->batch, 2 * sm_count()).total > kMaxSmemPerCta)
    return HGA_ERR_UNSUPPORTED;
  const int sms = sm_count();
  const SplitLayout lay(kv, p, sms);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  SplitArgs sp;
  sp.tiles = reinterpret_cast<uint32_t*>(ws + lay.tiles);
  sp.tile_stride = lay.tile_stride;
  sp.part = reinterpret_cast<float*>(ws + lay.part);
  sp.count = reinterpret_cast<int*>(ws + lay.count);
  sp.grid = split_grid(kv, p, sms);
  const int units = kv->batch * kv->n_kv_heads;
  const int P = pick_cluster(units);
  cudaError_t e = D == 128 ? launch_split<128>(a, sp, units, P, stream) : launch_split<64>(a, sp, units, P, stream);
  return e == cudaSuccess ? HGA_OK : HGA_ERR_CUDA;
}

int next_pow2(int x) {
  int p = 2;
  while (p < x) p <<= 1;
  return p;
}

// Fill the routing part of RoutedArgs (n_pad, kcap, params).
void routing_args(RoutedArgs& a, const hga_kv* kv, const hga_params* p) {
  const int nf_max = kv->max_len / p->chunk;
  const int cand_max = nf_max > 2 ? nf_max - 2 : 0;
  a.C = p->chunk;
  a.g = p->group;
  a.k = p->top_chunks;
  a.G = p->top_groups;
  a.n_pad = next_pow2(cand_max);
  const int kc = cand_max < p->top_chunks ? cand_max : p->top_chunks;
  a.kcap = kc < 1 ? 1 : kc;
}

// Routed tokens of one (block, head) when routing covers exactly [0, L).
int routed_count(int L, const hga_params* p) {
  const int C = p->chunk, nf = L / C;
  if (nf <= 2) return L;
  const int r = nf - 2 < p->top_chunks ? nf - 2 : p->top_chunks;
  return C + r * p->top_groups * p->group + (L - (nf - 1) * C);
}

// Shared checks of the prefill calls (batch 1, contiguous cache, head dim 128,
// blocks of 64 queries, 128-row tiles of two query heads).
hga_status check_prefill(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block, const hga_kv* kv,
                         int32_t cache_len, bool need_v) {
  hga_status s = check_kv(kv, need_v);
  if (s != HGA_OK) return s;
  if ((s = check_heads(n_q_heads, kv)) != HGA_OK) return s;
  if (q == nullptr || !aligned16(q) || n_queries < 1 || cache_len < 0) return HGA_ERR_INVALID_ARG;
  if ((int64_t)cache_len + n_queries > kv->max_len) return HGA_ERR_INVALID_ARG;
  if (kv->batch != 1 || kv->page_table != nullptr || kv->head_dim != 128) return HGA_ERR_UNSUPPORTED;
  if (block != kBlockQ || n_queries % block != 0) return HGA_ERR_UNSUPPORTED;
  if (((n_q_heads / kv->n_kv_heads) * block) % kPfRows != 0) return HGA_ERR_UNSUPPORTED;
  return HGA_OK;
}

hga_status launch_block_route(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                              const hga_kv* kv, int32_t cache_len, const void* chunk_sum, const void* group_sum,
                              const hga_params* p, int32_t* idx, int32_t idx_stride, int32_t* n_idx,
                              cudaStream_t stream, bool growing = false) {
  BlockRouteArgs a;
  std::memset(&a, 0, sizeof a);
  a.q = static_cast<const uint16_t*>(q);
  a.hq = n_q_heads;
  a.R = n_q_heads / kv->n_kv_heads;
  a.T = n_queries;
  a.block = block;
  a.chunk_sum = static_cast<const uint16_t*>(chunk_sum);
  a.group_sum = static_cast<const uint16_t*>(group_sum);
  a.hkv = kv->n_kv_heads;
  a.max_chunks = kv->max_len / p->chunk;
  a.L = cache_len;
  a.C = p->chunk;
  a.g = p->group;
  a.k = p->top_chunks;
  a.G = p->top_groups;
  a.idx = idx;
  a.n_idx = n_idx;
  a.idx_stride = idx_stride;
  a.growing = growing ? 1 : 0;
  const int n_pad = a.max_chunks - 2 > 2 ? a.max_chunks - 2 : 2;
  const int kcap_raw = a.max_chunks - 2 < a.k ? a.max_chunks - 2 : a.k;
  const int kcap = kcap_raw < 1 ? 1 : kcap_raw;
  const int smem = BlockRouteSmem(128, n_pad, kcap, a.G, a.C / a.g).total + 8 * n_pad;
  if (smem > kMaxSmemPerCta) return HGA_ERR_UNSUPPORTED;
  static std::atomic<int> smem_set[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HGA_ERR_CUDA;
  if (smem > smem_set[dev].load()) {
    if (cudaFuncSetAttribute(block_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return HGA_ERR_CUDA;
    smem_set[dev].store(smem);
  }
  const int units = (n_queries / block) * kv->n_kv_heads;
  block_route_kernel<<<units, kRoutedThreads, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? HGA_OK : HGA_ERR_CUDA;
}

hga_status launch_prefill_attend(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                                 const hga_kv* kv, int32_t cache_len, const int32_t* idx, int32_t idx_stride,
                                 const int32_t* n_idx, const hga_params* p, float* out, cudaStream_t stream,
                                 bool growing = false) {
  PrefillAttnArgs a;
  std::memset(&a, 0, sizeof a);
  a.q = static_cast<const uint16_t*>(q);
  a.hq = n_q_heads;
  a.R = n_q_heads / kv->n_kv_heads;
  a.T = n_queries;
  a.block = block;
  a.k = static_cast<const uint16_t*>(kv->k);
  a.v = static_cast<const uint16_t*>(kv->v);
  a.hkv = kv->n_kv_heads;
  a.max_len = kv->max_len;
  a.cache_len = cache_len;
  a.idx = idx;
  a.n_idx = n_idx;
  a.idx_stride = idx_stride;
  a.scale_log2 = scale_log2(p, kv->head_dim);
  a.out = out;
  a.growing = growing ? 1 : 0;
  a.fail_at_tile = g_fail_at_tile.load();
  static std::atomic<bool> configured[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HGA_ERR_CUDA;
  if (!configured[dev].load()) {
    if (cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PrefillSmem::kTotal) != cudaSuccess)
      return HGA_ERR_CUDA;
    // two CTAs per SM need the largest shared-memory carveout; this kernel
    // moves K/V with cp.async into shared memory, so a small L1 costs nothing
    if (cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) !=
        cudaSuccess)
      return HGA_ERR_CUDA;
    configured[dev].store(true);
  }
  const int m_tiles = a.R * block / kPfRows;
  const int grid = (n_queries / block) * kv->n_kv_heads * m_tiles;
  prefill_attn_kernel<<<grid, kPfThreads, PrefillSmem::kTotal, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? HGA_OK : HGA_ERR_CUDA;
}

// Routed-list area of hga_prefill_noalloc: a fixed device array that every GPU
// loading the library keeps until process exit, so that the entry point never
// allocates. Host code must not pass the symbol itself to a kernel (on the host
// it is only a stand-in); the device address comes from cudaGetSymbolAddress.
constexpr size_t kNoAllocPrefillBytes = 2u << 20;
static __device__ __align__(256) unsigned char g_noalloc_prefill_ws[kNoAllocPrefillBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_prefill_ws on the current device, looked up once
// per device (with that device current) and cached.
hga_status noalloc_area(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HGA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_prefill_ws) != cudaSuccess || ptr == nullptr) return HGA_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return HGA_OK;
}

template <int D>
cudaError_t launch_hisa(const RoutedArgs& a, int units, int P, int smem_bytes, cudaStream_t stream) {
  auto kern = hisa_decode_kernel<D>;
  static std::atomic<int> smem_set[kMaxDevices];
  static std::atomic<bool> np_set[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (smem_bytes > smem_set[dev].load()) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return e;
    smem_set[dev].store(smem_bytes);
  }
  if (P > 8 && !np_set[dev].load()) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    np_set[dev].store(true);
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3((unsigned)(units * P), 1, 1);
  cfg.blockDim = dim3(kRoutedThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// Kept tokens of the block-then-token route at the longest context (the list
// length hga_decode_hisa writes is at most this).
int hisa_max_routed(const hga_kv* kv, const hga_params* p, int32_t top_tokens) {
  const int C = p->chunk, nf = kv->max_len / C;
  int most = 0;  // most candidates over lengths <= max_len
  for (int L = kv->max_len; L >= 0 && L > kv->max_len - 2 * C; --L) {
    const int f = L / C;
    const int n = f <= 2 ? L : C + (f - 2 < p->top_chunks ? f - 2 : p->top_chunks) * C + (L - (f - 1) * C);
    if (n > most) most = n;
  }
  (void)nf;
  return most < top_tokens ? most : top_tokens;
}


// Floats of the logits workspace per (sequence, KV head): 8 per candidate of the
// token step, for the most candidates at any length.
int64_t hisa_logit_stride(const hga_kv* kv, const hga_params* p) {
  RoutedArgs a;
  std::memset(&a, 0, sizeof a);
  routing_args(a, kv, p);
  return (int64_t)hisa_tok_pad(p->chunk, a.kcap) * kMaxHeadsPerKv;
}

hga_status hisa_impl(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum, const hga_params* p,
                     int32_t top_tokens, float* out, float* lse, int32_t* idx, int32_t idx_stride, int32_t* n_idx,
                     float* logits, cudaStream_t stream) {
  hga_status s = check_kv(kv, true);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if ((s = check_heads(n_q_heads, kv)) != HGA_OK) return s;
  if (q == nullptr || !aligned16(q) || chunk_sum == nullptr || !aligned16(chunk_sum) || out == nullptr ||
      top_tokens < 1)
    return HGA_ERR_INVALID_ARG;
  if ((idx == nullptr) != (n_idx == nullptr)) return HGA_ERR_INVALID_ARG;
  if (idx != nullptr && idx_stride < hisa_max_routed(kv, p, top_tokens)) return HGA_ERR_INVALID_ARG;
  if (p->chunk % 16 != 0) return HGA_ERR_UNSUPPORTED;  // token batches of 16 stay inside one chunk
  RoutedArgs a;
  std::memset(&a, 0, sizeof a);
  a.kv = make_kv_view(kv);
  a.sv = make_sum_view(kv, p, chunk_sum, nullptr);
  a.q = static_cast<const uint16_t*>(q);
  a.hq = n_q_heads;
  a.R = n_q_heads / kv->n_kv_heads;
  routing_args(a, kv, p);
  // never more than the most candidates at any length: a larger top_tokens keeps every candidate
  // either way, and this bounds the shared-memory list
  a.k_tok = hisa_max_routed(kv, p, top_tokens);
  a.scale_log2 = scale_log2(p, kv->head_dim);
  a.out = out;
  a.lse = lse;
  a.idx_out = idx;
  a.n_idx_out = n_idx;
  a.idx_stride = idx ? idx_stride : 0;
  a.logits = logits;
  a.lg_stride = logits ? hisa_logit_stride(kv, p) : 0;
  const int smem = HisaSmem(kv->head_dim, a.n_pad, a.kcap, hisa_tok_pad(p->chunk, a.kcap), a.k_tok).total;
  if (smem > kMaxSmemPerCta) return HGA_ERR_UNSUPPORTED;
  const int units = kv->batch * kv->n_kv_heads;
  const int P = pick_cluster(units);
  cudaError_t e = kv->head_dim == 128 ? launch_hisa<128>(a, units, P, smem, stream)
                                      : launch_hisa<64>(a, units, P, smem, stream);
  return e == cudaSuccess ? HGA_OK : HGA_ERR_CUDA;
}

}  // namespace
}  // namespace hga

using namespace hga;

extern "C" {

const char* hga_status_string(hga_status s) {
  switch (s) {
    case HGA_OK: return "ok";
    case HGA_ERR_INVALID_ARG: return "invalid argument";
    case HGA_ERR_UNSUPPORTED: return "unsupported size or layout";
    case HGA_ERR_CUDA: return "CUDA runtime error";
    case HGA_ERR_DEVICE_FAULT: return "bad device-side input (skipped by the kernel)";
    case HGA_ERR_TIMEOUT: return "bounded device wait expired";
  }
  return "unknown status";
}

hga_status hga_summary_bytes(const hga_kv* kv, const hga_params* p, size_t* chunk_bytes,
                             size_t* group_bytes) {
  hga_status s = check_kv(kv, false);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  const size_t d = (size_t)kv->head_dim, gpc = (size_t)(p->chunk / p->group);
  const size_t slots = kv->page_table ? (size_t)kv->num_pages * kv->n_kv_heads
                                      : (size_t)kv->batch * kv->n_kv_heads * (kv->max_len / p->chunk);
  if (chunk_bytes) *chunk_bytes = slots * d * 2;
  if (group_bytes) *group_bytes = slots * gpc * d * 2;
  return HGA_OK;
}

int32_t hga_max_routed_tokens(const hga_kv* kv, const hga_params* p) {
  if (check_kv(kv, false) != HGA_OK || check_params(p, kv, true) != HGA_OK) return -1;
  return max_routed(kv, p);
}

hga_status hga_build_summaries(const hga_kv* kv, const hga_params* p, void* chunk_sum,
                               void* group_sum, cudaStream_t stream) {
  hga_status s = check_kv(kv, false);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if (chunk_sum == nullptr || group_sum == nullptr || !aligned16(chunk_sum) || !aligned16(group_sum))
    return HGA_ERR_INVALID_ARG;
  const int max_chunks = kv->max_len / p->chunk;
  if (max_chunks == 0) return HGA_OK;
  const int gpc = p->chunk / p->group;
  const KvView kvv = make_kv_view(kv);
  const SumView sv = make_sum_view(kv, p, chunk_sum, group_sum);
  dim3 grid((unsigned)max_chunks, (unsigned)kv->n_kv_heads, (unsigned)kv->batch);
  dim3 block((unsigned)(32 * (gpc < 8 ? gpc : 8)));
  const size_t smem = (size_t)gpc * kv->head_dim * sizeof(float);
  if (kv->head_dim == 128)
    summaries_kernel<128><<<grid, block, smem, stream>>>(kvv, sv, p->chunk, p->group, 0);
  else
    summaries_kernel<64><<<grid, block, smem, stream>>>(kvv, sv, p->chunk, p->group, 0);
  return cudaGetLastError() == cudaSuccess ? HGA_OK : HGA_ERR_CUDA;
}

hga_status hga_append(const hga_kv* kv, int32_t* seq_lens, const void* k_new, const void* v_new,
                      const hga_params* p, void* chunk_sum, void* group_sum, cudaStream_t stream) {
  hga_status s = check_kv(kv, true);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if (seq_lens == nullptr || seq_lens != kv->seq_lens || k_new == nullptr || v_new == nullptr ||
      !aligned16(k_new) || !aligned16(v_new) || chunk_sum == nullptr || group_sum == nullptr ||
      !aligned16(chunk_sum) || !aligned16(group_sum))
    return HGA_ERR_INVALID_ARG;
  const KvView kvv = make_kv_view(kv);
  const SumView sv = make_sum_view(kv, p, chunk_sum, group_sum);
  uint16_t* k = static_cast<uint16_t*>(const_cast<void*>(kv->k));
  uint16_t* v = static_cast<uint16_t*>(const_cast<void*>(kv->v));
  const uint16_t* kn = static_cast<const uint16_t*>(k_new);
  const uint16_t* vn = static_cast<const uint16_t*>(v_new);
  const int gpc = p->chunk / p->group;
  dim3 grid(1u, (unsigned)kv->n_kv_heads, (unsigned)kv->batch);
  dim3 block((unsigned)(32 * (gpc < 8 ? gpc : 8)));
  const size_t smem = (size_t)gpc * kv->head_dim * sizeof(float);
  if (kv->head_dim == 128) {
    append_kernel<128><<<kv->batch, 128, 0, stream>>>(kvv, k, v, seq_lens, kn, vn);
    summaries_kernel<128><<<grid, block, smem, stream>>>(kvv, sv, p->chunk, p->group, 1);
  } else {
    append_kernel<64><<<kv->batch, 128, 0, stream>>>(kvv, k, v, seq_lens, kn, vn);
    summaries_kernel<64><<<grid, block, smem, stream>>>(kvv, sv, p->chunk, p->group, 1);
  }
  return cudaGetLastError() == cudaSuccess ? HGA_OK : HGA_ERR_CUDA;
}

hga_status hga_route(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                     const void* group_sum, const hga_params* p, int32_t* idx, int32_t idx_stride,
                     int32_t* n_idx, cudaStream_t stream) {
  hga_status s = check_kv(kv, false);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if ((s = check_heads(n_q_heads, kv)) != HGA_OK) return s;
  if (q == nullptr || !aligned16(q) || chunk_sum == nullptr || group_sum == nullptr ||
      !aligned16(chunk_sum) || !aligned16(group_sum) || idx == nullptr || n_idx == nullptr)
    return HGA_ERR_INVALID_ARG;
  if (idx_stride < max_routed(kv, p)) return HGA_ERR_INVALID_ARG;
  RoutedArgs a;
  std::memset(&a, 0, sizeof a);
  a.kv = make_kv_view(kv);
  a.sv = make_sum_view(kv, p, chunk_sum, group_sum);
  a.q = static_cast<const uint16_t*>(q);
  a.hq = n_q_heads;
  a.R = n_q_heads / kv->n_kv_heads;
  routing_args(a, kv, p);
  a.scale_log2 = scale_log2(p, kv->head_dim);
  a.idx_out = idx;
  a.n_idx_out = n_idx;
  a.idx_stride = idx_stride;
  return run_routed<kModeRoute>(a, kv->head_dim, kv->batch * kv->n_kv_heads, stream);
}

hga_status hga_attend(const void* q, int32_t n_q_heads, const hga_kv* kv, const int32_t* idx,
                      int32_t idx_stride, const int32_t* n_idx, const hga_params* p, float* out,
                      float* lse, cudaStream_t stream) {
  hga_status s = check_kv(kv, true);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, false)) != HGA_OK) return s;
  if ((s = check_heads(n_q_heads, kv)) != HGA_OK) return s;
  if (q == nullptr || !aligned16(q) || idx == nullptr || n_idx == nullptr || out == nullptr ||
      idx_stride < 1)
    return HGA_ERR_INVALID_ARG;
  RoutedArgs a;
  std::memset(&a, 0, sizeof a);
  a.kv = make_kv_view(kv);
  a.sv = make_sum_view(kv, nullptr, nullptr, nullptr);
  a.q = static_cast<const uint16_t*>(q);
  a.hq = n_q_heads;
  a.R = n_q_heads / kv->n_kv_heads;
  a.C = a.g = a.k = a.G = 1;
  a.n_pad = 2;
  a.kcap = 1;
  a.scale_log2 = scale_log2(p, kv->head_dim);
  a.out = out;
  a.lse = lse;
  a.idx_in = idx;
  a.n_idx_in = n_idx;
  a.idx_stride = idx_stride;
  return run_routed<kModeAttend>(a, kv->head_dim, kv->batch * kv->n_kv_heads, stream);
}

static hga_status decode_impl(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                       const void* group_sum, const hga_params* p, float* out, float* lse, int32_t* idx,
                       int32_t idx_stride, int32_t* n_idx, void* workspace, cudaStream_t stream) {
  RoutedArgs a;
  std::memset(&a, 0, sizeof a);
  a.kv = make_kv_view(kv);
  a.sv = make_sum_view(kv, p, chunk_sum, group_sum);
  a.q = static_cast<const uint16_t*>(q);
  a.hq = n_q_heads;
  a.R = n_q_heads / kv->n_kv_heads;
  routing_args(a, kv, p);
  a.scale_log2 = scale_log2(p, kv->head_dim);
  a.out = out;
  a.lse = lse;
  a.idx_out = idx;
  a.n_idx_out = n_idx;
  a.idx_stride = idx ? idx_stride : 0;
  // The route + balanced attention pair is opt-in: on B200 the fused kernel is
  // faster at every batch measured (1, 4, 16 and 64 sequences of 64K tokens).
  const int choice = g_decode_kernel.load();
  if (workspace != nullptr && choice == 3 && split_applies(kv, p))
    return run_split(a, kv, p, workspace, kv->head_dim, stream);
  if (choice != 1 && p->group % 16 == 0)
    return run_decode(a, kv->head_dim, kv->batch * kv->n_kv_heads, stream);
  return run_routed<kModeDecode>(a, kv->head_dim, kv->batch * kv->n_kv_heads, stream);
}

static hga_status check_decode(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                        const void* group_sum, const hga_params* p, float* out, int32_t* idx, int32_t idx_stride,
                        int32_t* n_idx) {
  hga_status s = check_kv(kv, true);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if ((s = check_heads(n_q_heads, kv)) != HGA_OK) return s;
  if (q == nullptr || !aligned16(q) || chunk_sum == nullptr || group_sum == nullptr ||
      !aligned16(chunk_sum) || !aligned16(group_sum) || out == nullptr)
    return HGA_ERR_INVALID_ARG;
  if ((idx == nullptr) != (n_idx == nullptr)) return HGA_ERR_INVALID_ARG;
  if (idx != nullptr && idx_stride < max_routed(kv, p)) return HGA_ERR_INVALID_ARG;
  return HGA_OK;
}

hga_status hga_decode(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                      const void* group_sum, const hga_params* p, float* out, float* lse,
                      int32_t* idx, int32_t idx_stride, int32_t* n_idx, cudaStream_t stream) {
  hga_status s = check_decode(q, n_q_heads, kv, chunk_sum, group_sum, p, out, idx, idx_stride, n_idx);
  if (s != HGA_OK) return s;
  return decode_impl(q, n_q_heads, kv, chunk_sum, group_sum, p, out, lse, idx, idx_stride, n_idx, nullptr, stream);
}

size_t hga_decode_workspace_size(const hga_kv* kv, int32_t n_q_heads, const hga_params* p) {
  if (check_kv(kv, false) != HGA_OK || check_params(p, kv, true) != HGA_OK || check_heads(n_q_heads, kv) != HGA_OK)
    return 0;
  if (!split_applies(kv, p)) return 256;
  return SplitLayout(kv, p, sm_count()).total;
}

hga_status hga_decode_ws(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                         const void* group_sum, const hga_params* p, float* out, float* lse, int32_t* idx,
                         int32_t idx_stride, int32_t* n_idx, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
  hga_status s = check_decode(q, n_q_heads, kv, chunk_sum, group_sum, p, out, idx, idx_stride, n_idx);
  if (s != HGA_OK) return s;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return HGA_ERR_INVALID_ARG;
  if (workspace_bytes < hga_decode_workspace_size(kv, n_q_heads, p)) return HGA_ERR_INVALID_ARG;
  return decode_impl(q, n_q_heads, kv, chunk_sum, group_sum, p, out, lse, idx, idx_stride, n_idx, workspace,
                     stream);
}

int32_t hga_max_hisa_tokens(const hga_kv* kv, const hga_params* p, int32_t top_tokens) {
  if (check_kv(kv, false) != HGA_OK || check_params(p, kv, true) != HGA_OK || top_tokens < 1) return -1;
  return hisa_max_routed(kv, p, top_tokens);
}

hga_status hga_decode_hisa(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                           const hga_params* p, int32_t top_tokens, float* out, float* lse, int32_t* idx,
                           int32_t idx_stride, int32_t* n_idx, cudaStream_t stream) {
  return hisa_impl(q, n_q_heads, kv, chunk_sum, p, top_tokens, out, lse, idx, idx_stride, n_idx, nullptr, stream);
}

size_t hga_decode_hisa_workspace_size(const hga_kv* kv, const hga_params* p) {
  if (check_kv(kv, false) != HGA_OK || check_params(p, kv, true) != HGA_OK) return 0;
  return (size_t)kv->batch * kv->n_kv_heads * (size_t)hisa_logit_stride(kv, p) * sizeof(float);
}

hga_status hga_decode_hisa_ws(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                              const hga_params* p, int32_t top_tokens, float* out, float* lse, int32_t* idx,
                              int32_t idx_stride, int32_t* n_idx, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  const size_t need = hga_decode_hisa_workspace_size(kv, p);
  if (need == 0) return HGA_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < need)
    return HGA_ERR_INVALID_ARG;
  return hisa_impl(q, n_q_heads, kv, chunk_sum, p, top_tokens, out, lse, idx, idx_stride, n_idx,
                   static_cast<float*>(workspace), stream);
}

hga_status hga_route_blocks(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                            const hga_kv* kv, int32_t cache_len, const void* chunk_sum, const void* group_sum,
                            const hga_params* p, int32_t* idx, int32_t idx_stride, int32_t* n_idx,
                            cudaStream_t stream) {
  hga_status s = check_prefill(q, n_q_heads, n_queries, block, kv, cache_len, false);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if (chunk_sum == nullptr || group_sum == nullptr || !aligned16(chunk_sum) || !aligned16(group_sum) ||
      idx == nullptr || n_idx == nullptr)
    return HGA_ERR_INVALID_ARG;
  if (idx_stride < routed_count(cache_len, p)) return HGA_ERR_INVALID_ARG;
  return launch_block_route(q, n_q_heads, n_queries, block, kv, cache_len, chunk_sum, group_sum, p, idx,
                            idx_stride, n_idx, stream);
}

hga_status hga_prefill_attend(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                              const hga_kv* kv, int32_t cache_len, const int32_t* idx, int32_t idx_stride,
                              const int32_t* n_idx, const hga_params* p, float* out, cudaStream_t stream) {
  hga_status s = check_prefill(q, n_q_heads, n_queries, block, kv, cache_len, true);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, false)) != HGA_OK) return s;
  if (idx == nullptr || n_idx == nullptr || out == nullptr || idx_stride < 1) return HGA_ERR_INVALID_ARG;
  return launch_prefill_attend(q, n_q_heads, n_queries, block, kv, cache_len, idx, idx_stride, n_idx, p, out,
                               stream);
}

size_t hga_prefill_workspace_size(const hga_kv* kv, int32_t n_q_heads, int32_t n_queries, int32_t block,
                                  int32_t cache_len, const hga_params* p) {
  if (check_kv(kv, false) != HGA_OK || check_params(p, kv, true) != HGA_OK || block < 1 || n_queries < 1 ||
      n_q_heads < 1 || cache_len < 0)
    return 0;
  const size_t units = (size_t)((n_queries + block - 1) / block) * kv->n_kv_heads;
  const size_t stride = (size_t)routed_count(cache_len, p);
  return units * (stride + 1) * sizeof(int32_t);
}

hga_status hga_prefill(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block, const hga_kv* kv,
                       int32_t cache_len, const void* chunk_sum, const void* group_sum, const hga_params* p,
                       float* out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  hga_status s = check_prefill(q, n_q_heads, n_queries, block, kv, cache_len, true);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if (chunk_sum == nullptr || group_sum == nullptr || !aligned16(chunk_sum) || !aligned16(group_sum) ||
      out == nullptr || workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 3u) != 0)
    return HGA_ERR_INVALID_ARG;
  const size_t need = hga_prefill_workspace_size(kv, n_q_heads, n_queries, block, cache_len, p);
  if (workspace_bytes < need) return HGA_ERR_INVALID_ARG;
  const int stride = routed_count(cache_len, p);
  const int units = (n_queries / block) * kv->n_kv_heads;
  int32_t* idx = static_cast<int32_t*>(workspace);
  int32_t* n_idx = idx + (size_t)units * stride;
  s = launch_block_route(q, n_q_heads, n_queries, block, kv, cache_len, chunk_sum, group_sum, p, idx, stride,
                         n_idx, stream);
  if (s != HGA_OK) return s;
  return launch_prefill_attend(q, n_q_heads, n_queries, block, kv, cache_len, idx, stride, n_idx, p, out, stream);
}

// Routed count of the longest list over the blocks of a growing-history
// prefill (block b routes over [0, cache_len + b * block)); the count is not
// monotone in the length (the local chunk's tail shrinks at a chunk boundary).
int routed_count_growing(int32_t cache_len, int32_t n_queries, int32_t block, const hga_params* p) {
  int best = 0;
  for (int b = 0; b * block < n_queries; ++b) {
    const int c = routed_count(cache_len + b * block, p);
    if (c > best) best = c;
  }
  return best;
}

hga_status hga_route_blocks_growing(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                                    const hga_kv* kv, int32_t cache_len, const void* chunk_sum,
                                    const void* group_sum, const hga_params* p, int32_t* idx, int32_t idx_stride,
                                    int32_t* n_idx, cudaStream_t stream) {
  hga_status s = check_prefill(q, n_q_heads, n_queries, block, kv, cache_len, false);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if (chunk_sum == nullptr || group_sum == nullptr || !aligned16(chunk_sum) || !aligned16(group_sum) ||
      idx == nullptr || n_idx == nullptr)
    return HGA_ERR_INVALID_ARG;
  if (idx_stride < routed_count_growing(cache_len, n_queries, block, p)) return HGA_ERR_INVALID_ARG;
  return launch_block_route(q, n_q_heads, n_queries, block, kv, cache_len, chunk_sum, group_sum, p, idx,
                            idx_stride, n_idx, stream, true);
}

size_t hga_prefill_growing_workspace_size(const hga_kv* kv, int32_t n_q_heads, int32_t n_queries, int32_t block,
                                          int32_t cache_len, const hga_params* p) {
  if (check_kv(kv, false) != HGA_OK || check_params(p, kv, true) != HGA_OK || block < 1 || n_queries < 1 ||
      n_q_heads < 1 || cache_len < 0)
    return 0;
  const size_t units = (size_t)((n_queries + block - 1) / block) * kv->n_kv_heads;
  const size_t stride = (size_t)routed_count_growing(cache_len, n_queries, block, p);
  return units * (stride + 1) * sizeof(int32_t);
}

hga_status hga_prefill_growing(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                               const hga_kv* kv, int32_t cache_len, const void* chunk_sum, const void* group_sum,
                               const hga_params* p, float* out, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  hga_status s = check_prefill(q, n_q_heads, n_queries, block, kv, cache_len, true);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if (chunk_sum == nullptr || group_sum == nullptr || !aligned16(chunk_sum) || !aligned16(group_sum) ||
      out == nullptr || workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 3u) != 0)
    return HGA_ERR_INVALID_ARG;
  const size_t need = hga_prefill_growing_workspace_size(kv, n_q_heads, n_queries, block, cache_len, p);
  if (workspace_bytes < need) return HGA_ERR_INVALID_ARG;
  const int stride = routed_count_growing(cache_len, n_queries, block, p);
  const int units = (n_queries / block) * kv->n_kv_heads;
  int32_t* idx = static_cast<int32_t*>(workspace);
  int32_t* n_idx = idx + (size_t)units * stride;
  s = launch_block_route(q, n_q_heads, n_queries, block, kv, cache_len, chunk_sum, group_sum, p, idx, stride,
                         n_idx, stream, true);
  if (s != HGA_OK) return s;
  return launch_prefill_attend(q, n_q_heads, n_queries, block, kv, cache_len, idx, stride, n_idx, p, out, stream,
                               true);
}

hga_status hga_prefill_noalloc(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                               const hga_kv* kv, int32_t cache_len, const void* chunk_sum, const void* group_sum,
                               const hga_params* p, float* out, cudaStream_t stream) {
  hga_status s = check_prefill(q, n_q_heads, n_queries, block, kv, cache_len, true);
  if (s != HGA_OK) return s;
  if ((s = check_params(p, kv, true)) != HGA_OK) return s;
  if (chunk_sum == nullptr || group_sum == nullptr || !aligned16(chunk_sum) || !aligned16(group_sum) ||
      out == nullptr)
    return HGA_ERR_INVALID_ARG;
  if (hga_prefill_workspace_size(kv, n_q_heads, n_queries, block, cache_len, p) > kNoAllocPrefillBytes)
    return HGA_ERR_UNSUPPORTED;
  void* area = nullptr;
  if ((s = noalloc_area(&area)) != HGA_OK) return s;
  // Every list entry read later is written first by the routing kernel, so the
  // area needs no clearing between calls.
  const int stride = routed_count(cache_len, p);
  const int units = (n_queries / block) * kv->n_kv_heads;
  int32_t* idx = static_cast<int32_t*>(area);
  int32_t* n_idx = idx + (size_t)units * stride;
  s = launch_block_route(q, n_q_heads, n_queries, block, kv, cache_len, chunk_sum, group_sum, p, idx, stride,
                         n_idx, stream);
  if (s != HGA_OK) return s;
  return launch_prefill_attend(q, n_q_heads, n_queries, block, kv, cache_len, idx, stride, n_idx, p, out, stream);
}

hga_status hga_set_launch_option(int32_t option, int32_t value) {
  if (option == HGA_OPT_CTAS_PER_HEAD) {
    if (value < 0 || value > 16) return HGA_ERR_INVALID_ARG;
    g_ctas_per_head.store(value);
    return HGA_OK;
  }
  if (option == HGA_OPT_DECODE_KERNEL) {
    if (value < 0 || value > 3) return HGA_ERR_INVALID_ARG;
    g_decode_kernel.store(value);
    return HGA_OK;
  }
  if (option == HGA_OPT_TEST_EXPIRE_PREFILL_WAIT) {
    if (value < 0) return HGA_ERR_INVALID_ARG;
    g_fail_at_tile.store(value - 1);
    return HGA_OK;
  }
  return HGA_ERR_INVALID_ARG;
}

hga_status hga_host_kv_pointer(const void* host, void** device_ptr) {
  if (device_ptr == nullptr) return HGA_ERR_INVALID_ARG;
  *device_ptr = nullptr;
  if (host == nullptr) return HGA_ERR_INVALID_ARG;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, host) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of an unknown pointer
    return HGA_ERR_INVALID_ARG;
  }
  if (attr.type != cudaMemoryTypeHost) return HGA_ERR_INVALID_ARG;
  void* dev = nullptr;
  if (cudaHostGetDevicePointer(&dev, const_cast<void*>(host), 0) != cudaSuccess || dev == nullptr) {
    cudaGetLastError();
    return HGA_ERR_INVALID_ARG;
  }
  *device_ptr = dev;
  return HGA_OK;
}

hga_status hga_get_device_error(cudaStream_t stream, int32_t* bits) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return HGA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return HGA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess) return HGA_ERR_CUDA;
  }
  if (bits) *bits = v;
  if (v & kErrTimeout) return HGA_ERR_TIMEOUT;
  return v ? HGA_ERR_DEVICE_FAULT : HGA_OK;
}

}  // extern "C"
