/*
 * CPU oracle for Hierarchical Global Attention routed attention.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow, double-precision
 * statement of what the routed-attention path computes. Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg load it; the library never
 * does, and it shares no code with the CUDA kernels.
 *
 * Source of the method: "Hierarchical Global Attention (HGA)" (Woernle,
 * Fedosov, Grinenko; arXiv 2606.30709), abstract: a query scores per-chunk
 * summaries of the rotary-embedded keys and keeps the best chunks, narrows to
 * the best groups inside those chunks, and attends exactly to the tokens of the
 * kept groups. Keeping the start and the end of the context in every selection
 * follows the HISA article ("Hierarchical Indexing Sparse Attention",
 * shijienb.com summary, two-step block-then-token filter).
 *
 * Readings taken where the pages leave a step open (each is listed with its
 * reason in the design notes):
 *   - a chunk summary is the mean of the post-rotary keys of the chunk, a group
 *     summary the mean over one group; accumulated in double and rounded to
 *     bfloat16 (round to nearest, ties to even) for storage;
 *   - only full chunks get summaries; with nf = floor(L / C) full chunks,
 *     chunk 0 (sink) and chunk nf-1 plus the partial tail (local) are always
 *     kept whole and are not candidates; nf <= 2 means dense attention;
 *   - the routing score of a KV head is the sum over the query heads that share
 *     it, without the softmax scale; ties go to the lower index;
 *   - prefill blocks share one routing decision: the score is the maximum over
 *     the block's queries of the head-summed score;
 *   - the block-then-token variant (oracle_hisa_route) uses the chunks as its
 *     blocks and the same head-summed score for blocks and tokens; the first
 *     and last blocks are always among the kept blocks, and the token step
 *     chooses among all kept blocks' tokens.
 *
 * Parity pins for every function are in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bfloat16 */

/* bfloat16 bits -> double (exact). */
double oracle_bf16_to_double(uint16_t h) {
  uint32_t bits = (uint32_t)h << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/*
 * double -> bfloat16 bits with round to nearest, ties to even, taken directly
 * on the binary64 pattern (no intermediate float rounding).
 * bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits.
 */
uint16_t oracle_bf16_rne(double x) {
  uint64_t u;
  memcpy(&u, &x, sizeof u);
  uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
  int64_t exp = (int64_t)((u >> 52) & 0x7FF);
  uint64_t frac = u & 0xFFFFFFFFFFFFFULL;
  if (exp == 0x7FF) return frac ? (uint16_t)0x7FC0 : (uint16_t)(sign | 0x7F80); /* NaN / inf */
  if (exp == 0 && frac == 0) return sign;                                       /* +-0 */
  /* value = sig * 2^(e2) with sig a 53-bit integer */
  uint64_t sig = exp ? (frac | (1ULL << 52)) : frac;
  int64_t e2 = exp ? exp - 1075 : -1074;
  /* bfloat16 keeps 8 significant bits for normals (exponent >= -126) and a fixed
   * quantum of 2^-133 below. Pick the quantum q = 2^qe of the result. */
  int64_t top = 0; /* index of the highest set bit of sig */
  for (int64_t b = 63; b >= 0; --b)
    if (sig >> b & 1) { top = b; break; }
  int64_t unbiased = e2 + top; /* x in [2^unbiased, 2^(unbiased+1)) */
  int64_t qe = unbiased >= -126 ? unbiased - 7 : -133;
  /* n = round_half_even(sig * 2^(e2 - qe)) */
  int64_t shift = qe - e2; /* bits to drop */
  uint64_t n;
  if (shift <= 0) {
    n = sig << (-shift);
  } else if (shift >= 64) {
    n = 0;
  } else {
    uint64_t keep = sig >> shift;
    uint64_t rem = sig & ((1ULL << shift) - 1);
    uint64_t half = 1ULL << (shift - 1);
    n = keep + ((rem > half || (rem == half && (keep & 1))) ? 1 : 0);
  }
  /* re-normalise: n may have grown to 2^8 (normal) or reached 2^7 (subnormal -> normal) */
  if (n == 0) return sign;
  int64_t nb = 0;
  for (int64_t b = 63; b >= 0; --b)
    if (n >> b & 1) { nb = b; break; }
  int64_t value_exp = qe + nb; /* n * 2^qe in [2^value_exp, 2^(value_exp+1)) */
  if (value_exp > 127) return (uint16_t)(sign | 0x7F80);
  if (value_exp < -126) {
    /* subnormal: stored fraction = n (quantum 2^-133) */
    return (uint16_t)(sign | (uint16_t)n);
  }
  uint16_t bexp = (uint16_t)(value_exp + 127);
  /* align the leading one to bit 7 (n has 8 or 9 significant bits here) and drop it */
  uint64_t aligned = nb >= 7 ? (n >> (nb - 7)) : (n << (7 - nb));
  uint16_t bfrac = (uint16_t)(aligned & 0x7F);
  return (uint16_t)(sign | (bexp << 7) | bfrac);
}

/* ------------------------------------------------------------- summaries */

/*
 * Chunk and group summaries of one (sequence, KV head).
 *   K          [L][d] bfloat16 bits, post-rotary keys, row stride d
 *   chunk_sum  [nf][d]        bfloat16: s_c = (1/C) sum_{t in chunk c} K_t
 *   group_sum  [nf][C/g][d]   bfloat16: s_{c,j} = (1/g) sum_{t in group j of c} K_t
 *   *_f64      optional unrounded double copies (may be NULL)
 * nf = floor(L / C): the partial tail gets no summary.
 */
void oracle_summaries(const uint16_t* K, int32_t L, int32_t d, int32_t C, int32_t g,
                      uint16_t* chunk_sum, uint16_t* group_sum, double* chunk_f64,
                      double* group_f64) {
  int32_t nf = L / C, gpc = C / g;
  for (int32_t c = 0; c < nf; ++c) {
    for (int32_t e = 0; e < d; ++e) {
      double acc = 0.0;
      for (int32_t t = c * C; t < (c + 1) * C; ++t) acc += oracle_bf16_to_double(K[(int64_t)t * d + e]);
      double mean = acc / (double)C;
      chunk_sum[(int64_t)c * d + e] = oracle_bf16_rne(mean);
      if (chunk_f64) chunk_f64[(int64_t)c * d + e] = mean;
    }
    for (int32_t j = 0; j < gpc; ++j)
      for (int32_t e = 0; e < d; ++e) {
        double acc = 0.0;
        int32_t t0 = c * C + j * g;
        for (int32_t t = t0; t < t0 + g; ++t) acc += oracle_bf16_to_double(K[(int64_t)t * d + e]);
        double mean = acc / (double)g;
        int64_t o = ((int64_t)c * gpc + j) * d + e;
        group_sum[o] = oracle_bf16_rne(mean);
        if (group_f64) group_f64[o] = mean;
      }
  }
}

/* ---------------------------------------------------------------- scoring */

/*
 * Routing score of one summary vector s for a block of n_q queries of one KV
 * head: max over queries p of sum over the R query heads i of q_{p,i} . s.
 * q is [n_q][q_row_stride] with head i of query p at q + p*q_row_stride + i*d.
 * For a single decode query (n_q = 1) this is the head-summed score.
 */
static double route_score(const uint16_t* q, int32_t n_q, int64_t q_row_stride, int32_t R,
                          int32_t d, const uint16_t* s) {
  double best = -INFINITY;
  for (int32_t p = 0; p < n_q; ++p) {
    double acc = 0.0;
    for (int32_t i = 0; i < R; ++i) {
      const uint16_t* qi = q + (int64_t)p * q_row_stride + (int64_t)i * d;
      for (int32_t e = 0; e < d; ++e) acc += oracle_bf16_to_double(qi[e]) * oracle_bf16_to_double(s[e]);
    }
    if (acc > best) best = acc;
  }
  return best;
}

/* Scores of all nf chunk summaries (chunk_sum [nf][d]). */
void oracle_chunk_scores(const uint16_t* q, int32_t n_q, int64_t q_row_stride, int32_t R, int32_t d,
                         const uint16_t* chunk_sum, int32_t nf, double* out) {
  for (int32_t c = 0; c < nf; ++c) out[c] = route_score(q, n_q, q_row_stride, R, d, chunk_sum + (int64_t)c * d);
}

/* Scores of the gpc group summaries of one chunk (group_sum_chunk [gpc][d]). */
void oracle_group_scores(const uint16_t* q, int32_t n_q, int64_t q_row_stride, int32_t R, int32_t d,
                         const uint16_t* group_sum_chunk, int32_t gpc, double* out) {
  for (int32_t j = 0; j < gpc; ++j)
    out[j] = route_score(q, n_q, q_row_stride, R, d, group_sum_chunk + (int64_t)j * d);
}

/* ---------------------------------------------------------------- routing */

typedef struct {
  double score;
  int32_t id;
} scored;

/* Higher score first; equal scores: lower id first. */
static int by_score_desc(const void* a, const void* b) {
  const scored* x = (const scored*)a;
  const scored* y = (const scored*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->id > y->id) - (x->id < y->id);
}

static int by_int_asc(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/*
 * Two-level routing of one (sequence, KV head) for a block of n_q queries.
 *   chunk_sum [nf][d], group_sum [nf][C/g][d]: bfloat16 summaries of the first
 *   nf = floor(L/C) chunks.
 * Writes the routed token positions, ascending, to tokens (capacity cap) and
 * returns their number; -1 if cap is too small. Optionally writes the kept
 * middle chunks (ascending) to kept_chunks and returns their count in *n_kept.
 *
 *   nf <= 2          -> every token [0, L)
 *   otherwise        -> [0, C)  (sink chunk)
 *                       + for each of the top min(k, nf-2) chunks among 1..nf-2,
 *                         its top min(G, C/g) groups
 *                       + [(nf-1)*C, L)  (local chunk and partial tail)
 */
int32_t oracle_route_block(const uint16_t* q, int32_t n_q, int64_t q_row_stride, int32_t R, int32_t d,
                           const uint16_t* chunk_sum, const uint16_t* group_sum, int32_t L,
                           int32_t C, int32_t g, int32_t k, int32_t G, int32_t* tokens, int32_t cap,
                           int32_t* kept_chunks, int32_t* n_kept) {
  int32_t nf = L / C, gpc = C / g;
  int32_t n = 0;
  if (n_kept) *n_kept = 0;
  if (nf <= 2) {
    if (L > cap) return -1;
    for (int32_t t = 0; t < L; ++t) tokens[n++] = t;
    return n;
  }
  int32_t n_cand = nf - 2;
  int32_t r = k < n_cand ? k : n_cand;
  int32_t gk = G < gpc ? G : gpc;
  int64_t need = (int64_t)C + (int64_t)r * gk * g + (L - (int64_t)(nf - 1) * C);
  if (need > cap) return -1;

  scored* cand = (scored*)malloc(sizeof(scored) * (size_t)n_cand);
  int32_t* chosen = (int32_t*)malloc(sizeof(int32_t) * (size_t)(r > 0 ? r : 1));
  scored* grp = (scored*)malloc(sizeof(scored) * (size_t)gpc);
  int32_t* gsel = (int32_t*)malloc(sizeof(int32_t) * (size_t)gpc);
  for (int32_t c = 1; c <= nf - 2; ++c) {
    cand[c - 1].score = route_score(q, n_q, q_row_stride, R, d, chunk_sum + (int64_t)c * d);
    cand[c - 1].id = c;
  }
  qsort(cand, (size_t)n_cand, sizeof(scored), by_score_desc);
  for (int32_t i = 0; i < r; ++i) chosen[i] = cand[i].id;
  qsort(chosen, (size_t)r, sizeof(int32_t), by_int_asc);

  for (int32_t t = 0; t < C; ++t) tokens[n++] = t; /* sink */
  for (int32_t i = 0; i < r; ++i) {
    int32_t c = chosen[i];
    for (int32_t j = 0; j < gpc; ++j) {
      grp[j].score = route_score(q, n_q, q_row_stride, R, d, group_sum + ((int64_t)c * gpc + j) * d);
      grp[j].id = j;
    }
    qsort(grp, (size_t)gpc, sizeof(scored), by_score_desc);
    for (int32_t m = 0; m < gk; ++m) gsel[m] = grp[m].id;
    qsort(gsel, (size_t)gk, sizeof(int32_t), by_int_asc);
    for (int32_t m = 0; m < gk; ++m)
      for (int32_t t = 0; t < g; ++t) tokens[n++] = c * C + gsel[m] * g + t;
  }
  for (int32_t t = (nf - 1) * C; t < L; ++t) tokens[n++] = t; /* local + tail */

  if (kept_chunks) memcpy(kept_chunks, chosen, sizeof(int32_t) * (size_t)r);
  if (n_kept) *n_kept = r;
  free(cand);
  free(chosen);
  free(grp);
  free(gsel);
  return n;
}

/* Decode routing: one query, its R heads at q[0..R*d). */
int32_t oracle_route(const uint16_t* q, int32_t R, int32_t d, const uint16_t* chunk_sum,
                     const uint16_t* group_sum, int32_t L, int32_t C, int32_t g, int32_t k, int32_t G,
                     int32_t* tokens, int32_t cap) {
  return oracle_route_block(q, 1, (int64_t)R * d, R, d, chunk_sum, group_sum, L, C, g, k, G, tokens,
                            cap, NULL, NULL);
}

/* ------------------------------------------------- block-then-token routing */

/*
 * Block-then-token routing of one decode query (the HISA article's two steps,
 * "Hierarchical Indexing Sparse Attention", shijienb.com summary: a coarse
 * filter on per-block feature vectors keeps the best blocks, always with the
 * start and the end of the text, then token-level scoring runs only inside the
 * kept blocks). Blocks are the chunks of size C with the same summaries, and the
 * scoring rule is the head-summed one of oracle_route:
 *   nf <= 2 -> candidates: every token [0, L)
 *   else    -> candidates: [0, C) (first block) + the tokens of the top
 *              min(m, nf-2) chunks among 1..nf-2 (score desc, id asc) +
 *              [(nf-1)*C, L) (last block and partial tail)
 *   token score tau_t = sum over the R heads of q_i . K_t (double); keep the
 *   top min(k_tok, n_cand) candidates by (tau desc, t asc), written ascending.
 *   K [L][d] holds the keys of this (sequence, KV head).
 * Returns the kept count, -1 if cap is too small. *n_scored (optional) gets the
 * number of scored vectors (the cost the article's O(L^2/B + L m B) counts over
 * a whole prefill): (nf - 2) summaries + n_cand tokens when nf > 2, n_cand
 * otherwise.
 */
int32_t oracle_hisa_route(const uint16_t* q, int32_t R, int32_t d, const uint16_t* chunk_sum, const uint16_t* K,
                          int32_t L, int32_t C, int32_t m, int32_t k_tok, int32_t* tokens, int32_t cap,
                          int64_t* n_scored) {
  int32_t nf = L / C;
  int32_t* cand_tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
  int32_t n_cand = 0;
  int64_t scored_vectors = 0;
  if (nf <= 2) {
    for (int32_t t = 0; t < L; ++t) cand_tok[n_cand++] = t;
  } else {
    int32_t n_blk = nf - 2;
    int32_t r = m < n_blk ? m : n_blk;
    scored* blk = (scored*)malloc(sizeof(scored) * (size_t)n_blk);
    int32_t* chosen = (int32_t*)malloc(sizeof(int32_t) * (size_t)(r > 0 ? r : 1));
    for (int32_t c = 1; c <= nf - 2; ++c) {
      blk[c - 1].score = route_score(q, 1, (int64_t)R * d, R, d, chunk_sum + (int64_t)c * d);
      blk[c - 1].id = c;
    }
    scored_vectors += n_blk;
    qsort(blk, (size_t)n_blk, sizeof(scored), by_score_desc);
    for (int32_t i = 0; i < r; ++i) chosen[i] = blk[i].id;
    qsort(chosen, (size_t)r, sizeof(int32_t), by_int_asc);
    for (int32_t t = 0; t < C; ++t) cand_tok[n_cand++] = t; /* first block */
    for (int32_t i = 0; i < r; ++i)
      for (int32_t t = 0; t < C; ++t) cand_tok[n_cand++] = chosen[i] * C + t;
    for (int32_t t = (nf - 1) * C; t < L; ++t) cand_tok[n_cand++] = t; /* last block + tail */
    free(blk);
    free(chosen);
  }
  scored_vectors += n_cand;
  if (n_scored) *n_scored = scored_vectors;
  int32_t keep = k_tok < n_cand ? k_tok : n_cand;
  if (keep > cap) {
    free(cand_tok);
    return -1;
  }
  scored* tok = (scored*)malloc(sizeof(scored) * (size_t)(n_cand > 0 ? n_cand : 1));
  for (int32_t i = 0; i < n_cand; ++i) {
    tok[i].score = route_score(q, 1, (int64_t)R * d, R, d, K + (int64_t)cand_tok[i] * d);
    tok[i].id = cand_tok[i];
  }
  qsort(tok, (size_t)n_cand, sizeof(scored), by_score_desc);
  for (int32_t i = 0; i < keep; ++i) tokens[i] = tok[i].id;
  qsort(tokens, (size_t)keep, sizeof(int32_t), by_int_asc);
  free(tok);
  free(cand_tok);
  return keep;
}

/* -------------------------------------------------------------- attention */

/*
 * Exact softmax attention of R query heads over a token set.
 *   q [R][d], K and V [*][d] (row t is token t), tokens[n] positions.
 *   out [R][d]: o_i = sum_t softmax_t(scale * q_i . K_t) V_t
 *   lse [R] (optional): natural log of sum_t exp(scale * q_i . K_t)
 * n == 0 gives out = 0 and lse = -inf.
 */
void oracle_attend(const uint16_t* q, int32_t R, int32_t d, const uint16_t* K, const uint16_t* V,
                   const int32_t* tokens, int32_t n, double scale, double* out, double* lse) {
  double* z = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  for (int32_t i = 0; i < R; ++i) {
    const uint16_t* qi = q + (int64_t)i * d;
    double* oi = out + (int64_t)i * d;
    for (int32_t e = 0; e < d; ++e) oi[e] = 0.0;
    if (n == 0) {
      if (lse) lse[i] = -INFINITY;
      continue;
    }
    double m = -INFINITY;
    for (int32_t a = 0; a < n; ++a) {
      const uint16_t* kt = K + (int64_t)tokens[a] * d;
      double acc = 0.0;
      for (int32_t e = 0; e < d; ++e) acc += oracle_bf16_to_double(qi[e]) * oracle_bf16_to_double(kt[e]);
      z[a] = acc * scale;
      if (z[a] > m) m = z[a];
    }
    double den = 0.0;
    for (int32_t a = 0; a < n; ++a) {
      double w = exp(z[a] - m);
      den += w;
      const uint16_t* vt = V + (int64_t)tokens[a] * d;
      for (int32_t e = 0; e < d; ++e) oi[e] += w * oracle_bf16_to_double(vt[e]);
    }
    for (int32_t e = 0; e < d; ++e) oi[e] /= den;
    if (lse) lse[i] = m + log(den);
  }
  free(z);
}

/*
 * Chunked-prefill block of one KV head: n_q queries at positions P .. P+n_q-1
 * share the routed cache set cache_tokens[n_cache]; query p additionally sees
 * the block's own tokens P .. P+p (causal).
 *   q [n_q][q_row_stride] (R heads of d at q + p*q_row_stride + i*d)
 *   K, V [*][d] hold the cache and the block's own tokens at their positions.
 *   out [n_q][R][d]
 */
void oracle_prefill_block(const uint16_t* q, int32_t n_q, int64_t q_row_stride, int32_t R, int32_t d,
                          const uint16_t* K, const uint16_t* V, const int32_t* cache_tokens,
                          int32_t n_cache, int32_t P, double scale, double* out) {
  int32_t* tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_cache + n_q));
  memcpy(tok, cache_tokens, sizeof(int32_t) * (size_t)n_cache);
  uint16_t* qrow = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)R * d);
  for (int32_t p = 0; p < n_q; ++p) {
    for (int32_t t = 0; t <= p; ++t) tok[n_cache + t] = P + t;
    for (int32_t i = 0; i < R; ++i)
      memcpy(qrow + (int64_t)i * d, q + (int64_t)p * q_row_stride + (int64_t)i * d, sizeof(uint16_t) * (size_t)d);
    oracle_attend(qrow, R, d, K, V, tok, n_cache + p + 1, scale, out + (int64_t)p * R * d, NULL);
  }
  free(qrow);
  free(tok);
}
