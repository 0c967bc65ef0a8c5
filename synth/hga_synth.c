/*
 * Seeded synthetic inputs for routed-attention decode and prefill.
 *
 * This module only MAKES inputs: Gaussian K, V and q, rotary position embedding
 * applied to K and q, and "planted" chunks whose keys are shifted toward the
 * query direction. It holds none of the routing or attention arithmetic, and it
 * is shared by the CPU oracle and the GPU path so that both see identical bytes.
 *
 * Random numbers: SplitMix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014) used as a counter-based
 * generator: value n of stream s is mix(key(seed, s) + (n + 1) * golden), so any
 * element can be produced independently and in parallel. Normals come from the
 * Box-Muller transform on two 53-bit uniforms in (0, 1).
 *
 * Rotary embedding: rotate-half layout (dimension e pairs with e + d/2),
 * frequency theta^(-2e/d), applied in double precision.
 *
 * Every tensor is rounded once, at the end, to bfloat16 with round-to-nearest-
 * even.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Raw 64-bit draw n of stream `stream` under `seed`. */
uint64_t synth_u64(uint64_t seed, uint64_t stream, uint64_t n) {
  uint64_t key = sm64_mix(seed * SYNTH_GOLDEN + sm64_mix(stream + SYNTH_GOLDEN));
  return sm64_mix(key + (n + 1) * SYNTH_GOLDEN);
}

static inline double u01_open(uint64_t x) {
  /* 53-bit uniform strictly inside (0, 1). */
  return ((double)(x >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* Standard normal draw n of stream `stream` (Box-Muller, cosine branch). */
double synth_normal(uint64_t seed, uint64_t stream, uint64_t n) {
  double u1 = u01_open(synth_u64(seed, stream, 2 * n));
  double u2 = u01_open(synth_u64(seed, stream, 2 * n + 1));
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* double -> bfloat16 bits, round to nearest, ties to even. */
uint16_t synth_bf16_rne(double x) {
  if (isnan(x)) return (uint16_t)0x7FC0;
  double ax = fabs(x), r;
  if (ax == 0.0) {
    r = 0.0;
  } else if (ax < 0x1p-126) {
    /* bfloat16 subnormal range: spacing 2^-133. */
    r = nearbyint(ax * 0x1p133) * 0x1p-133;
  } else {
    int e;
    double m = frexp(ax, &e); /* ax = m * 2^e, m in [0.5, 1) */
    r = ldexp(nearbyint(ldexp(m, 8)), e - 8); /* keep 8 significant bits */
  }
  float f = (float)r; /* exact (or +inf past the bfloat16 range) */
  uint32_t bits;
  memcpy(&bits, &f, sizeof bits);
  uint16_t h = (uint16_t)(bits >> 16);
  if (signbit(x)) h |= 0x8000;
  return h;
}

static inline double bf16_bits_to_double(uint16_t h) {
  uint32_t bits = (uint32_t)h << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* In-place rotate-half rotary embedding of one d-vector at position pos. */
static void rope_inplace(double* x, int32_t d, double pos, double theta) {
  int32_t half = d / 2;
  for (int32_t e = 0; e < half; ++e) {
    double freq = pow(theta, -(2.0 * (double)e) / (double)d);
    double ang = pos * freq;
    double c = cos(ang), s = sin(ang);
    double x1 = x[e], x2 = x[e + half];
    x[e] = x1 * c - x2 * s;
    x[e + half] = x2 * c + x1 * s;
  }
}

enum { STREAM_Q = 0, STREAM_K = 1, STREAM_V = 2, STREAM_PLANT = 3, STREAMS_PER_SEQ = 8 };

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/*
 * Draw n_plant distinct chunk ids from [1, n_chunks - 2] by a partial
 * Fisher-Yates shuffle; ascending on return. Returns the count drawn (0 when
 * there are fewer than 3 chunks).
 */
int32_t synth_plant_chunks(uint64_t seed, int32_t seq, int32_t n_chunks, int32_t n_plant,
                           int32_t* out) {
  if (n_chunks < 3 || n_plant <= 0) return 0;
  int32_t n = n_chunks - 2;
  if (n_plant > n) n_plant = n;
  int32_t* a = (int32_t*)malloc(sizeof(int32_t) * (size_t)n);
  if (!a) return -1;
  for (int32_t i = 0; i < n; ++i) a[i] = i + 1;
  uint64_t stream = (uint64_t)seq * STREAMS_PER_SEQ + STREAM_PLANT;
  for (int32_t i = 0; i < n_plant; ++i) {
    uint64_t span = (uint64_t)(n - i);
    int32_t j = i + (int32_t)(synth_u64(seed, stream, (uint64_t)i) % span);
    int32_t t = a[i];
    a[i] = a[j];
    a[j] = t;
  }
  memcpy(out, a, sizeof(int32_t) * (size_t)n_plant);
  free(a);
  qsort(out, (size_t)n_plant, sizeof(int32_t), cmp_i32);
  return n_plant;
}

/*
 * One sequence of synthetic inputs.
 *
 *   q_out  [n_q][Hq][d]  bf16: N(0,1), rotary at q_pos[p]
 *   k_out  [Hkv][L][d]   bf16: N(0,1), rotary at t, plus 0.5 * u_h on planted chunks
 *   v_out  [Hkv][L][d]   bf16: N(0,1)
 * Head h of K/V starts at k_out + h * kv_head_stride (elements), so the caller
 * can write straight into a wider [Hkv][Lmax][d] buffer.
 *
 * u_h is the unit vector along the sum, over all n_q queries and the Hq/Hkv query
 * heads that share KV head h, of the bf16-rounded post-rotary q. Planted chunks
 * are drawn from [1, plant_chunks - 2]; chunk c covers tokens [c*chunk, (c+1)*chunk).
 * Returns the number of planted chunks written to planted_out (may be NULL).
 */
int32_t synth_sequence(uint64_t seed, int32_t seq, int32_t L, int32_t n_q, const int32_t* q_pos,
                       int32_t Hq, int32_t Hkv, int32_t d, double theta, int32_t chunk,
                       int32_t plant_chunks, int32_t n_plant, uint16_t* q_out, uint16_t* k_out,
                       uint16_t* v_out, int64_t kv_head_stride, int32_t* planted_out) {
  if (L < 0 || n_q < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || (d & 1) || Hq % Hkv) return -1;
  int32_t R = Hq / Hkv;
  uint64_t base = (uint64_t)seq * STREAMS_PER_SEQ;

  /* q */
  double* qd = (double*)malloc(sizeof(double) * (size_t)((int64_t)(n_q > 0 ? n_q : 1) * Hq * d));
  if (!qd) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t pi = 0; pi < (int64_t)n_q * Hq; ++pi) {
    int32_t p = (int32_t)(pi / Hq);
    double* x = qd + pi * d;
    for (int32_t e = 0; e < d; ++e) x[e] = synth_normal(seed, base + STREAM_Q, (uint64_t)(pi * d + e));
    rope_inplace(x, d, (double)q_pos[p], theta);
    for (int32_t e = 0; e < d; ++e) {
      uint16_t h = synth_bf16_rne(x[e]);
      q_out[pi * d + e] = h;
      x[e] = bf16_bits_to_double(h);
    }
  }

  /* planting direction per KV head */
  double* u = (double*)calloc((size_t)Hkv * d, sizeof(double));
  if (!u) { free(qd); return -1; }
  for (int32_t h = 0; h < Hkv; ++h) {
    double* uh = u + (int64_t)h * d;
    for (int32_t p = 0; p < n_q; ++p)
      for (int32_t i = 0; i < R; ++i) {
        const double* x = qd + ((int64_t)p * Hq + h * R + i) * d;
        for (int32_t e = 0; e < d; ++e) uh[e] += x[e];
      }
    double nrm = 0.0;
    for (int32_t e = 0; e < d; ++e) nrm += uh[e] * uh[e];
    nrm = sqrt(nrm);
    for (int32_t e = 0; e < d; ++e) uh[e] = nrm > 0.0 ? uh[e] / nrm : 0.0;
  }
  free(qd);

  int32_t n_planted = 0;
  int32_t* planted = NULL;
  unsigned char* is_planted = NULL;
  int32_t n_chunk_flags = chunk > 0 ? (L + chunk - 1) / chunk : 0;
  if (n_plant > 0 && chunk > 0) {
    planted = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_plant);
    is_planted = (unsigned char*)calloc((size_t)(n_chunk_flags > 0 ? n_chunk_flags : 1), 1);
    if (!planted || !is_planted) { free(u); free(planted); free(is_planted); return -1; }
    n_planted = synth_plant_chunks(seed, seq, plant_chunks, n_plant, planted);
    for (int32_t i = 0; i < n_planted; ++i)
      if (planted[i] < n_chunk_flags) is_planted[planted[i]] = 1;
    if (planted_out) memcpy(planted_out, planted, sizeof(int32_t) * (size_t)n_planted);
  }

  /* K and V */
#pragma omp parallel for schedule(static)
  for (int64_t ht = 0; ht < (int64_t)Hkv * L; ++ht) {
    int32_t h = (int32_t)(ht / L), t = (int32_t)(ht % L);
    double x[512];
    double* xs = d <= 512 ? x : (double*)malloc(sizeof(double) * (size_t)d);
    uint64_t n0 = (uint64_t)ht * (uint64_t)d;
    for (int32_t e = 0; e < d; ++e) xs[e] = synth_normal(seed, base + STREAM_K, n0 + (uint64_t)e);
    rope_inplace(xs, d, (double)t, theta);
    if (is_planted && is_planted[t / chunk]) {
      const double* uh = u + (int64_t)h * d;
      for (int32_t e = 0; e < d; ++e) xs[e] += 0.5 * uh[e];
    }
    uint16_t* kr = k_out + (int64_t)h * kv_head_stride + (int64_t)t * d;
    uint16_t* vr = v_out + (int64_t)h * kv_head_stride + (int64_t)t * d;
    for (int32_t e = 0; e < d; ++e) kr[e] = synth_bf16_rne(xs[e]);
    for (int32_t e = 0; e < d; ++e) vr[e] = synth_bf16_rne(synth_normal(seed, base + STREAM_V, n0 + (uint64_t)e));
    if (xs != x) free(xs);
  }

  free(u);
  free(planted);
  free(is_planted);
  return n_planted;
}

/* Seeded Fisher-Yates permutation of [0, n). */
void synth_permutation(uint64_t seed, uint64_t stream, int32_t n, int32_t* out) {
  for (int32_t i = 0; i < n; ++i) out[i] = i;
  for (int32_t i = n - 1; i > 0; --i) {
    int32_t j = (int32_t)(synth_u64(seed, stream, (uint64_t)i) % (uint64_t)(i + 1));
    int32_t t = out[i];
    out[i] = out[j];
    out[j] = t;
  }
}

/* Seeded integers, uniform over [lo, hi] inclusive. */
void synth_uniform_ints(uint64_t seed, uint64_t stream, int32_t n, int32_t lo, int32_t hi,
                        int32_t* out) {
  uint64_t span = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
  for (int32_t i = 0; i < n; ++i) out[i] = lo + (int32_t)(synth_u64(seed, stream, (uint64_t)i) % span);
}
