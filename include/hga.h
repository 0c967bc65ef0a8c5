/*
 * hga.h - C ABI of the routed-attention library (libhga.so), sm_100a.
 *
 * The method: "Hierarchical Global Attention (HGA)" (Woernle, Fedosov,
 * Grinenko; arXiv 2606.30709), abstract. A drop-in replacement for dense causal
 * attention with the pretrained projections unchanged: a query first scores
 * compact summaries of fixed-size key chunks and keeps the best chunks, then
 * scores per-group summaries inside them and keeps the best groups, then runs
 * exact softmax attention over the routed tokens only. The first chunk (sink)
 * and the last chunk with any partial tail (local) are always kept, following
 * the keep-beginning-and-end rule of the HISA article ("Hierarchical Indexing
 * Sparse Attention", shijienb.com summary, two-step block-then-token filter).
 *
 * The library takes post-projection, post-rotary q and K (the caller applies the
 * rotary embedding) plus V, and returns the attention output before the output
 * projection.
 *
 * Conventions shared by every call:
 *   - All data pointers are DEVICE pointers owned by the caller, except the
 *     hga_kv / hga_params structs themselves, which are read on the host during
 *     the call and may be freed on return.
 *   - bfloat16 tensors are passed as raw 16-bit patterns (`const void*`), 16-byte
 *     aligned; int32/float tensors are naturally aligned.
 *   - Calls are asynchronous on `stream`. The library allocates no device
 *     memory; its state is one device error word per device (a __device__
 *     variable), the fixed routed-list array of hga_prefill_noalloc, and a
 *     process-wide launch option (hga_set_launch_option).
 *   - Host validation failures return HGA_ERR_INVALID_ARG or
 *     HGA_ERR_UNSUPPORTED synchronously with nothing enqueued. Problems only the
 *     device can see (a sequence length above max_len, a page id outside the
 *     pool, a token index outside its sequence) make the kernel skip the
 *     offending access and set the device error word, read and cleared by
 *     hga_get_device_error. No kernel traps.
 *
 * Supported sizes: head_dim 64 or 128; n_q_heads % n_kv_heads == 0 with at most
 * 8 query heads per KV head; chunk % group == 0, chunk / group <= 32;
 * floor(max_len / chunk) <= 4096; 1 <= top_groups <= chunk / group;
 * top_chunks >= 1. Routing tables live in shared memory: parameter sets whose
 * tables (about 4 * min(top_chunks, max_len/chunk) * (top_groups + chunk/group + 2)
 * bytes) do not fit in shared memory next to the working buffers return
 * HGA_ERR_UNSUPPORTED.
 */
#ifndef HGA_H_
#define HGA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HGA_OK = 0,
  HGA_ERR_INVALID_ARG = 1,  /* bad pointer, size or parameter; nothing enqueued */
  HGA_ERR_UNSUPPORTED = 2,  /* valid but outside the supported sizes above; nothing enqueued */
  HGA_ERR_CUDA = 3,         /* a CUDA runtime call failed (see cudaGetLastError) */
  HGA_ERR_DEVICE_FAULT = 4, /* a kernel met a bad device-side input and skipped it */
  HGA_ERR_TIMEOUT = 5       /* a bounded device wait ran out */
} hga_status;

/*
 * Routing parameters. The paper's abstract fixes the two-level order (chunks,
 * then groups) but not the sizes; these are the caller's choice.
 */
typedef struct {
  int32_t chunk;      /* C: tokens per chunk (one summary per full chunk) */
  int32_t group;      /* g: tokens per group, chunk % group == 0 */
  int32_t top_chunks; /* k: routed chunks kept among chunks 1 .. nf-2 */
  int32_t top_groups; /* G: groups kept in each routed chunk */
  float scale;        /* softmax scale; 0 means 1/sqrt(head_dim). Routing never scales. */
} hga_params;

/*
 * The key/value cache.
 *   Contiguous (page_table == NULL): k, v are [batch][n_kv_heads][max_len][head_dim].
 *   Paged: k, v are a page pool [num_pages][n_kv_heads][page_size][head_dim];
 *   token t of sequence b sits in page page_table[b * max_pages + t / page_size]
 *   at row t % page_size. Paged caches require page_size == chunk, so one page is
 *   one chunk and summaries are indexed by physical page.
 * seq_lens[b] (device) is the number of valid tokens of sequence b, at most max_len.
 * A decode query of sequence b sits at position seq_lens[b] - 1; its own key and
 * value are already in the cache.
 */
typedef struct {
  const void* k;
  const void* v;
  const int32_t* page_table; /* device, [batch][max_pages], or NULL */
  const int32_t* seq_lens;   /* device, [batch] */
  int32_t batch;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t max_len;
  int32_t page_size; /* paged only */
  int32_t max_pages; /* paged only: page-table row length, max_pages * page_size >= max_len */
  int32_t num_pages; /* paged only: pages in the pool */
} hga_kv;

/*
 * Summary buffers (bfloat16), written by hga_build_summaries, read by routing.
 *   Contiguous: chunk_sum [batch][n_kv_heads][max_len/chunk][head_dim]
 *               group_sum [batch][n_kv_heads][max_len/chunk][chunk/group][head_dim]
 *   Paged:      chunk_sum [num_pages][n_kv_heads][head_dim]
 *               group_sum [num_pages][n_kv_heads][chunk/group][head_dim]
 * hga_summary_bytes reports both sizes.
 */
hga_status hga_summary_bytes(const hga_kv* kv, const hga_params* p, size_t* chunk_bytes,
                             size_t* group_bytes);

/*
 * Build chunk and group summaries from the post-rotary keys (the abstract's
 * per-chunk summaries, which see positions through the rotary embedding).
 * Summary of chunk c: the mean of
 * K_t over t in [c*C, (c+1)*C); of group j of chunk c: the mean over
 * [c*C + j*g, c*C + (j+1)*g). fp32 accumulation, bfloat16 round-to-nearest
 * store. Only full chunks (c < seq_lens[b] / C) are written; other entries are
 * left untouched. One pass over K; run it after filling the cache.
 */
hga_status hga_build_summaries(const hga_kv* kv, const hga_params* p, void* chunk_sum,
                               void* group_sum, cudaStream_t stream);

/*
 * Append one token to every sequence and keep the summaries current, for a
 * decode loop that grows the cache (the incremental form of the summaries
 * above; the pages keep summaries of the cached context up to date as it
 * grows). For every sequence b:
 *   K/V row k_new[b][h], v_new[b][h] -> position L = seq_lens[b] (contiguous
 *   row, or slot L / page_size of the page table, whose page the caller has
 *   assigned); then seq_lens[b] = L + 1, on the device; then, if L + 1 is a
 *   multiple of chunk, the summaries of the chunk just completed, with the
 *   same arithmetic as hga_build_summaries (bit-identical results).
 *   k_new, v_new  [batch][n_kv_heads][head_dim] bfloat16, device
 *   seq_lens      must be kv->seq_lens (updated in place)
 * Two kernels on `stream`, no host synchronisation and no allocation, so the
 * call can be captured in a CUDA graph together with hga_decode (call it once
 * before capturing so its launch attributes are set). A sequence already at
 * max_len is reported (device error bit 1) and left unchanged.
 */
hga_status hga_append(const hga_kv* kv, int32_t* seq_lens, const void* k_new, const void* v_new,
                      const hga_params* p, void* chunk_sum, void* group_sum, cudaStream_t stream);

/*
 * Upper bound on the routed tokens of one (sequence, KV head) over every
 * sequence length up to kv->max_len: the minimum idx_stride for hga_route,
 * hga_attend and hga_decode. Returns -1 on invalid arguments.
 */
int32_t hga_max_routed_tokens(const hga_kv* kv, const hga_params* p);

/*
 * Two-level routing (abstract: chunks are picked by their summaries first, then
 * only the best groups inside the picked chunks are kept). Per sequence b and
 * KV head h, with the R = n_q_heads /
 * n_kv_heads query heads i of h, nf = seq_lens[b] / chunk full chunks:
 *   nf <= 2: every token [0, L) is routed.
 *   else: chunk score sigma_c = sum_i q_i . s_c over candidates c in [1, nf-2];
 *         keep the top_chunks highest (ties: lower c); inside each kept chunk
 *         group score tau_{c,j} = sum_i q_i . s_{c,j}, keep the top_groups highest
 *         (ties: lower j); token list = [0, C) + kept groups (ascending) +
 *         [(nf-1)*C, L).
 *   q       [batch][n_q_heads][head_dim] bfloat16, post-rotary
 *   idx     [batch][n_kv_heads][idx_stride] int32 out: routed positions, ascending
 *   n_idx   [batch][n_kv_heads] int32 out: number of routed positions
 * idx_stride must be >= hga_max_routed_tokens(kv, p).
 */
hga_status hga_route(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                     const void* group_sum, const hga_params* p, int32_t* idx, int32_t idx_stride,
                     int32_t* n_idx, cudaStream_t stream);

/*
 * Exact softmax attention over a given token set (abstract: attention over the
 * routed tokens is exact, not approximated). For every query head i of KV head h:
 *   out[b][i] = sum_t softmax_t(scale * q_i . K_t) V_t over t in idx[b][h][0:n_idx]
 *   lse[b][i] = log sum_t exp(scale * q_i . K_t)    (natural log; lse may be NULL)
 * The R query heads of a KV head share every K/V tile. An empty set gives
 * out = 0 and lse = -inf. Tokens must lie in [0, seq_lens[b]); others are skipped
 * and reported through the device error word.
 *   out [batch][n_q_heads][head_dim] float32, lse [batch][n_q_heads] float32.
 * Only p->scale is read from p.
 */
hga_status hga_attend(const void* q, int32_t n_q_heads, const hga_kv* kv, const int32_t* idx,
                      int32_t idx_stride, const int32_t* n_idx, const hga_params* p, float* out,
                      float* lse, cudaStream_t stream);

/*
 * Fused decode step: hga_route followed by hga_attend in one kernel, the
 * routed positions kept on chip. idx / n_idx are optional outputs (both NULL,
 * or both set with idx_stride >= hga_max_routed_tokens).
 */
hga_status hga_decode(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                      const void* group_sum, const hga_params* p, float* out, float* lse,
                      int32_t* idx, int32_t idx_stride, int32_t* n_idx, cudaStream_t stream);

/*
 * Bytes of workspace hga_decode_ws needs for this cache and these parameters (0
 * on invalid arguments). The size depends on the current device's SM count:
 * query it with the device that will run the decode current.
 */
size_t hga_decode_workspace_size(const hga_kv* kv, int32_t n_q_heads, const hga_params* p);

/*
 * hga_decode with a caller-provided workspace (device memory, 256-byte aligned,
 * at least hga_decode_workspace_size bytes; its contents on entry do not matter
 * and on return are unspecified). Same arguments and results as hga_decode.
 * With a workspace the decode can run as two kernels that balance the
 * attention over the whole GPU (HGA_OPT_DECODE_KERNEL = 3): a route kernel
 * (the chunk scores, chunk top-k and group top-G of hga_route, one
 * thread-block cluster per (sequence, KV head)) writes the routed 16-token
 * tiles of every (sequence, KV head) into the workspace, and an attention
 * kernel cuts the tiles of all of them into equal slices, one per CTA,
 * merging the softmax partials of a (sequence, KV head) that several CTAs
 * share through the workspace. That pair applies when group % 16 == 0 and
 * batch <= 4096. By default (option 0) the call runs hga_decode's kernel,
 * which is faster on B200 at every batch measured, and leaves the workspace
 * unused. Calls that share one workspace must not overlap on the GPU.
 */
hga_status hga_decode_ws(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                         const void* group_sum, const hga_params* p, float* out, float* lse, int32_t* idx,
                         int32_t idx_stride, int32_t* n_idx, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/*
 * Chunked prefill. n_queries new tokens sit at positions cache_len ..
 * cache_len + n_queries - 1; their keys and values are already written into
 * the cache at those positions (kv->max_len >= cache_len + n_queries). The
 * queries are cut into blocks of `block` consecutive queries. Supported: batch 1,
 * contiguous cache, head_dim 128, block 64, n_queries % block == 0, and an even
 * number of query heads per KV head (two heads x 64 queries per 128-row tile).
 * kv->seq_lens is not read by the prefill calls; cache_len is given directly.
 * Summaries must cover the cache's full chunks (hga_build_summaries with
 * seq_lens[0] = cache_len).
 *
 * Block-shared routing (the prefill reading of the abstract's two-level
 * routing): for block b and KV head h, chunk scores are
 *   sigma_c = max over the block's queries p of sum_i q_{p,i} . s_c
 * and group scores likewise; the kept chunks, groups, sink and local chunk of
 * the cache [0, cache_len) follow hga_route. The scores are computed on tensor
 * cores with the head-summed queries split into a bf16 high part and a bf16
 * remainder (about 2^-16 relative error).
 *   idx   [n_queries/block][n_kv_heads][idx_stride] int32 out: routed cache positions
 *   n_idx [n_queries/block][n_kv_heads] int32 out
 * idx_stride must be >= the routed count for cache_len (hga_max_routed_tokens
 * of a cache with max_len = cache_len bounds it).
 */
hga_status hga_route_blocks(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                            const hga_kv* kv, int32_t cache_len, const void* chunk_sum, const void* group_sum,
                            const hga_params* p, int32_t* idx, int32_t idx_stride, int32_t* n_idx,
                            cudaStream_t stream);

/*
 * Prefill attention over given routed cache sets (abstract: exact attention over
 * the retrieved tokens): query p of block b (position P + p, P = cache_len + 64 b)
 * attends, for each of its query heads, to the cache positions idx[b][h][0:n_idx]
 * plus the block's own positions P .. P + p. Tensor-core (tcgen05) contraction
 * with fp32 accumulation in tensor memory.
 *   q [n_queries][n_q_heads][128] bf16, out [n_queries][n_q_heads][128] float32.
 * Only p->scale is read from p.
 */
hga_status hga_prefill_attend(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                              const hga_kv* kv, int32_t cache_len, const int32_t* idx, int32_t idx_stride,
                              const int32_t* n_idx, const hga_params* p, float* out, cudaStream_t stream);

/* Bytes of workspace hga_prefill needs (0 on invalid arguments). */
size_t hga_prefill_workspace_size(const hga_kv* kv, int32_t n_q_heads, int32_t n_queries, int32_t block,
                                  int32_t cache_len, const hga_params* p);

/*
 * hga_route_blocks followed by hga_prefill_attend; the routed lists live in the
 * caller's workspace (device memory, 4-byte aligned, at least
 * hga_prefill_workspace_size bytes; its contents on return are unspecified).
 */
hga_status hga_prefill(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block, const hga_kv* kv,
                       int32_t cache_len, const void* chunk_sum, const void* group_sum, const hga_params* p,
                       float* out, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * hga_prefill for callers that cannot allocate device memory. (The paper has no
 * counterpart; this is a property of the library.) Some callers have no way to
 * hand the library a workspace: a plugin whose host framework owns every device
 * allocation and gives the plugin no allocator, or a caller that must keep
 * cudaMalloc (which may synchronise the device) out of its serving loop. This
 * entry point allocates nothing and takes no workspace: the routed lists go to a
 * 2 MiB array of device memory inside the library, which every GPU that loads
 * the library holds until the process exits.
 *   - Same arguments and results as hga_prefill, without the workspace.
 *   - Limit: hga_prefill_workspace_size(...) must be at most 2 MiB (for example
 *     2048 queries in blocks of 64 with 4 KV heads and 2304 routed tokens uses
 *     1.18 MB); larger problems return HGA_ERR_UNSUPPORTED with nothing enqueued.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - All calls on a device share the one array, and it keeps the previous
 *     call's contents (nothing in it needs clearing: every entry that is read is
 *     written first by the same call). Calls whose execution overlaps on the GPU
 *     (different streams without ordering) race on it: order them.
 */
hga_status hga_prefill_noalloc(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                               const hga_kv* kv, int32_t cache_len, const void* chunk_sum, const void* group_sum,
                               const hga_params* p, float* out, cudaStream_t stream);

/*
 * Block-then-token routed decode, after the HISA article (shijienb.com news page
 * on Hierarchical Indexing Sparse Attention): its "step one, block-level coarse
 * filter" section scores one feature vector per fixed-size block and keeps the
 * best blocks, always with the beginning and the end of the text, then scores
 * tokens only inside the kept blocks; its advantages paragraph gives the
 * indexer cost going from O(L^2) to O(L^2/B + L m B). Blocks are the
 * chunks, with the summaries of hga_build_summaries (only chunk_sum is read),
 * and both steps use the head-summed score of hga_route. Per sequence b and KV
 * head h with nf = seq_lens[b] / chunk full chunks:
 *   candidates = every token [0, L) when nf <= 2; else [0, C) + the tokens of
 *   the top p->top_chunks chunks among 1..nf-2 (score desc, lower id first)
 *   + [(nf-1)*C, L)
 *   kept = the top_tokens candidates by tau_t = sum_i q_i . K_t (desc, lower
 *   position first), all of them if there are no more than top_tokens
 *   out/lse = exact softmax attention over the kept tokens, as hga_attend.
 * idx/n_idx (optional, as hga_decode) receive the kept positions, ascending;
 * idx_stride >= hga_max_hisa_tokens(kv, p, top_tokens). p->group and
 * p->top_groups must be valid as for hga_route but are not used. p->chunk must
 * be a multiple of 16, and the token keys of the most candidates at any length
 * ((min(top_chunks, max_len / chunk - 2) + 3) * chunk of them, 8 bytes each)
 * plus the kept list (4 bytes per kept token) must fit one CTA's 227 KB of
 * shared memory with the rest of its state (about 37 KB at head_dim 128);
 * HGA_ERR_UNSUPPORTED otherwise.
 */
hga_status hga_decode_hisa(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                           const hga_params* p, int32_t top_tokens, float* out, float* lse, int32_t* idx,
                           int32_t idx_stride, int32_t* n_idx, cudaStream_t stream);

/* Most positions hga_decode_hisa keeps for one (sequence, KV head); -1 on invalid arguments. */
int32_t hga_max_hisa_tokens(const hga_kv* kv, const hga_params* p, int32_t top_tokens);

/*
 * hga_decode_hisa with a caller-owned workspace (device memory, 256-byte
 * aligned, at least hga_decode_hisa_workspace_size bytes, used by this call
 * only). The token step then computes the per-head logits q_i . K_t of every
 * candidate with tensor-core tiles, keeps them in the workspace (fp32,
 * 32 bytes per candidate), takes tau_t as their sum over the query heads, and
 * the attention over the kept tokens reads those logits and the kept V rows,
 * not the kept K rows a second time. Same routing definition and outputs as
 * hga_decode_hisa (tau_t is summed in another order, which can change the
 * kept set only between near-equal scores). HGA_ERR_INVALID_ARG for a missing,
 * misaligned or short workspace; otherwise as hga_decode_hisa.
 */
hga_status hga_decode_hisa_ws(const void* q, int32_t n_q_heads, const hga_kv* kv, const void* chunk_sum,
                              const hga_params* p, int32_t top_tokens, float* out, float* lse, int32_t* idx,
                              int32_t idx_stride, int32_t* n_idx, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/*
 * Workspace bytes of hga_decode_hisa_ws: batch * n_kv_heads * 32 bytes per
 * candidate of the longest context ((min(top_chunks, max_len / chunk - 2) + 3)
 * * chunk candidates). 0 on invalid arguments.
 */
size_t hga_decode_hisa_workspace_size(const hga_kv* kv, const hga_params* p);

/*
 * Growing-history chunked prefill: the same calls as hga_route_blocks /
 * hga_prefill / hga_prefill_workspace_size, except that block b (queries at
 * P_b = cache_len + b * block .. P_b + block - 1) routes over everything before
 * it, [0, P_b), including the earlier blocks of the same call: its candidates
 * are the full chunks of [0, P_b), its local chunk the last of them plus the
 * partial tail up to P_b. Every query then attends its block's routed set plus
 * the block's own tokens up to itself (causal), so the result is the decode
 * rule applied block by block, as a drop-in for dense causal attention needs.
 * Summaries must cover the full chunks of [0, cache_len + n_queries - block)
 * (hga_build_summaries with seq_lens[0] = cache_len + n_queries, or hga_append
 * as the tokens arrive). idx_stride / the workspace are sized for the longest
 * list over the blocks (hga_prefill_growing_workspace_size).
 */
hga_status hga_route_blocks_growing(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                                    const hga_kv* kv, int32_t cache_len, const void* chunk_sum,
                                    const void* group_sum, const hga_params* p, int32_t* idx, int32_t idx_stride,
                                    int32_t* n_idx, cudaStream_t stream);
size_t hga_prefill_growing_workspace_size(const hga_kv* kv, int32_t n_q_heads, int32_t n_queries, int32_t block,
                                          int32_t cache_len, const hga_params* p);
hga_status hga_prefill_growing(const void* q, int32_t n_q_heads, int32_t n_queries, int32_t block,
                               const hga_kv* kv, int32_t cache_len, const void* chunk_sum, const void* group_sum,
                               const hga_params* p, float* out, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/*
 * Launch tuning, process-wide (not thread-safe against concurrent calls).
 *   HGA_OPT_CTAS_PER_HEAD: CTAs (one thread-block cluster) that cooperate on one
 *   (sequence, KV head) in hga_route / hga_attend / hga_decode; 0 = automatic,
 *   1..16 otherwise (above 8 needs non-portable cluster support).
 *   HGA_OPT_DECODE_KERNEL: which kernels run hga_decode / hga_decode_ws. 0 =
 *   automatic (the fused kernel that routes groups inside the attention warps
 *   when group % 16 == 0, else the phase-by-phase kernel), 1 = always the
 *   phase-by-phase kernel (the one hga_route and hga_attend use), 2 = the
 *   fused kernel where it applies, 3 = the route + balanced attention pair
 *   where it applies (hga_decode_ws only; elsewhere as 0). All compute the
 *   same routed set and attention.
 *   HGA_OPT_TEST_EXPIRE_PREFILL_WAIT: a test hook for the failure path of the
 *   prefill attention kernel. 0 = off (the default). v > 0 makes every CTA of
 *   the next prefill attention launches treat its wait for key tile v - 1 (its
 *   QK^T MMA) as expired AFTER that wait has really completed, so the kernel
 *   takes its timeout exit with no MMA outstanding: it stops issuing, waits for
 *   what it committed, releases tensor memory, writes no output row and
 *   reports HGA_ERR_TIMEOUT (error bit 8) through hga_get_device_error.
 *   Keep it 0 outside tests.
 * The options are process-wide by design: they choose launch shapes for tuning
 * and tests, not results (every choice computes the same routed set and
 * attention, except the test hook, which only makes calls fail).
 * Returns HGA_ERR_INVALID_ARG for an unknown option or value.
 */
enum { HGA_OPT_CTAS_PER_HEAD = 1, HGA_OPT_DECODE_KERNEL = 2, HGA_OPT_TEST_EXPIRE_PREFILL_WAIT = 4 };
hga_status hga_set_launch_option(int32_t option, int32_t value);

/*
 * Host-resident K/V (the pages' own placement: the full cache in host memory,
 * only the routed working set moved to the GPU). K and V may live in pinned,
 * mapped host memory (cudaHostAlloc, or cudaHostRegister with the mapped
 * flag); this call returns the device address of such a buffer, to be put in
 * hga_kv.k / hga_kv.v. The routing summaries stay in device memory. Every call
 * then reads K/V through the host link (PCIe or NVLink-C2C): hga_decode and
 * hga_route / hga_attend read only the routed rows, hga_build_summaries and
 * hga_append read and write what they always do. Returns HGA_ERR_INVALID_ARG
 * (and *device_ptr = NULL) when `host` is not pinned and mapped for the
 * current device, so an unmapped address never reaches a kernel.
 */
hga_status hga_host_kv_pointer(const void* host, void** device_ptr);

/*
 * Synchronise `stream`, then read and clear this device's error word.
 * HGA_OK if no kernel reported a problem since the last call,
 * HGA_ERR_DEVICE_FAULT for a bad device-side input, HGA_ERR_TIMEOUT for an
 * expired bounded wait, HGA_ERR_CUDA if the synchronisation itself failed.
 * `bits` (may be NULL) receives the raw word: 1 sequence length, 2 page id,
 * 4 token index, 8 timeout.
 */
hga_status hga_get_device_error(cudaStream_t stream, int32_t* bits);

/* Static description of a status code. */
const char* hga_status_string(hga_status s);

#ifdef __cplusplus
}
#endif

#endif /* HGA_H_ */
