/*
 * ORACLE -- test infrastructure only.  Nothing in the product path may call,
 * link or load this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code with the GPU path.
 *
 * What it computes: single-token paged-KV decode attention, the problem stated
 * in "spec(BACKEND-ROCM): the ROCm head_dim=128 decode arm, the ROCm half of
 * #382" (vllm.cpp PR #564, section "The gap it specs": bf16 decode attention
 * over a paged KV cache for GQA models) and in "perf(rocke): prepare saved
 * paged decode bindings once" (rocm-libraries PR #13700, section "Summary":
 * one-token split-KV attention, optional LSE output).  The pages print no
 * formula; their statement that a warp-strided online softmax differs from the
 * sequential kernel only by reduction order (PR #564, section "It is a mirror
 * of merged work, not new design") means the result is ordinary softmax
 * attention, and PR #13700 ("Testing Summary") checks against an independent
 * FP32 reference.  So the oracle is that definition, written out in double:
 *
 *   for every sequence b and query head h, with kv head kh = h / (Hq/Hkv):
 *     token t (0 <= t < L_b) lives in physical block block_tables[b][t / bs],
 *       slot t % bs:   k_t = K[phys, kh, slot, :],  v_t = V[phys, kh, slot, :]
 *     s_t   = scale * sum_d q[b,h,d] * k_t[d]
 *     M     = max_t s_t,  Z = sum_t exp(s_t - M)
 *     out   = sum_t exp(s_t - M) * v_t / Z
 *     lse   = M + ln Z                    (natural log, includes `scale`)
 *   L_b = 0 gives out = 0 and lse = -inf.
 *
 * Two options of the decode path that "Attention parity: run every attention
 * type on the best available path on both targets" (section "Current state")
 * lists next to dense GQA:
 *   sliding window W > 0: only tokens t >= L_b - W take part (the last W
 *     tokens; all of them when W >= L_b);
 *   attention sinks: a per-head logit sigma_h, in the units of s_t, joins the
 *     softmax with a zero value row:  M = max(max_t s_t, sigma_h),
 *     Z = sum_t exp(s_t - M) + exp(sigma_h - M); out and lse as above.  With
 *     L_b = 0: out = 0, lse = sigma_h.
 *
 * The cache may also hold 8-bit codes: "perf(rocke): prepare saved paged
 * decode bindings once" (sections "Summary" and the review's item N1) names an
 * FP8 decode path beside the non-FP8 one but fixes no format or scale.  The
 * reading taken: OCP FP8 E4M3 codes (OCP 8-bit Floating Point Specification,
 * E4M3: sign bit 7, exponent bits 6..3 with bias 7, mantissa bits 2..0,
 * exponent 0 for the subnormals m/8 * 2^-6, S.1111.111 is NaN, no infinities,
 * largest finite value 448) and one scale per tensor:
 *     k_t[d] = k_scale * E4M3(K code),  v_t[d] = v_scale * E4M3(V code),
 * after which everything above applies unchanged.  A bf16 cache is the same
 * with both scales 1.
 *
 * Exact two-pass softmax: no splits, no online rescaling.  bf16 inputs are
 * widened exactly to double.  Strides are in elements; every dimension may be
 * strided.  Work is spread over (b, kh) pairs with pthreads, which changes no
 * arithmetic order inside a pair.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t bits) {
  uint32_t w = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &w, 4);
  return (double)f;
}

/* The value of an E4M3 code, from the format's definition (header). */
static double e4m3_to_double(uint8_t code) {
  const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    mag = ldexp((double)m / 8.0, -6);
  else
    mag = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -mag : mag;
}

typedef struct {
  const uint16_t *q;
  const void *k;      /* bf16 bits (uint16) or E4M3 codes (uint8) */
  const void *v;
  int kv_fp8;         /* 0: bf16 cache; 1: E4M3 cache */
  double k_scale, v_scale;
  const int32_t *tables;
  const int32_t *lens;
  int64_t B, Hq, Hkv, D, bs, table_width;
  int64_t q_str[3];   /* b, h, d */
  int64_t kv_str[4];  /* block, kv head, slot, d (same for K and V) */
  double scale;
  int64_t window;     /* 0: every token; W > 0: the last W tokens */
  const float *sinks; /* NULL, or sink logit per query head [Hq] */
  double *out;        /* [B, Hq, D] contiguous */
  double *lse;        /* [B, Hq] */
} problem;

/* Element idx of a K or V cache, widened exactly to double, times the
 * tensor's scale. */
static double kv_value(const problem *p, const void *cache, int64_t idx, double tensor_scale) {
  if (p->kv_fp8) return tensor_scale * e4m3_to_double(((const uint8_t *)cache)[idx]);
  return tensor_scale * bf16_to_double(((const uint16_t *)cache)[idx]);
}

/* One query head of one sequence: the definition above, term by term. */
static void attend_one(const problem *p, int64_t b, int64_t h, double *s, double *o, double *lse) {
  const int64_t g = p->Hq / p->Hkv;
  const int64_t kh = h / g;
  const int64_t L = p->lens[b];
  const uint16_t *qrow = p->q + b * p->q_str[0] + h * p->q_str[1];
  const int has_sink = p->sinks != NULL;
  const double sink = has_sink ? (double)p->sinks[h] : 0.0;
  for (int64_t d = 0; d < p->D; ++d) o[d] = 0.0;
  if (L <= 0) {
    *lse = has_sink ? sink : -INFINITY;
    return;
  }
  /* the tokens that take part: [lo, L) */
  const int64_t lo = (p->window > 0 && L > p->window) ? L - p->window : 0;
  /* scores, s[t - lo] for token t */
  for (int64_t t = lo; t < L; ++t) {
    int64_t phys = p->tables[b * p->table_width + t / p->bs];
    int64_t slot = t % p->bs;
    const int64_t krow = phys * p->kv_str[0] + kh * p->kv_str[1] + slot * p->kv_str[2];
    double acc = 0.0;
    for (int64_t d = 0; d < p->D; ++d)
      acc += bf16_to_double(qrow[d * p->q_str[2]]) * kv_value(p, p->k, krow + d * p->kv_str[3], p->k_scale);
    s[t - lo] = p->scale * acc;
  }
  const int64_t n = L - lo;
  /* exact softmax (the sink, if any, joins the max and the denominator) */
  double M = s[0];
  for (int64_t t = 1; t < n; ++t)
    if (s[t] > M) M = s[t];
  if (has_sink && sink > M) M = sink;
  double Z = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    s[t] = exp(s[t] - M);
    Z += s[t];
  }
  if (has_sink) Z += exp(sink - M);
  /* weighted sum of values (the sink's value row is zero) */
  for (int64_t t = lo; t < L; ++t) {
    int64_t phys = p->tables[b * p->table_width + t / p->bs];
    int64_t slot = t % p->bs;
    const int64_t vrow = phys * p->kv_str[0] + kh * p->kv_str[1] + slot * p->kv_str[2];
    double w = s[t - lo] / Z;
    for (int64_t d = 0; d < p->D; ++d) o[d] += w * kv_value(p, p->v, vrow + d * p->kv_str[3], p->v_scale);
  }
  *lse = M + log(Z);
}

typedef struct {
  const problem *p;
  const int32_t *pairs; /* NULL: all (b, h); else npairs (b, h) pairs */
  int64_t npairs;
  int64_t max_len;
  int nthreads, tid;
} job;

static void *worker(void *arg) {
  job *j = (job *)arg;
  const problem *p = j->p;
  double *s = (double *)malloc(sizeof(double) * (size_t)(j->max_len > 0 ? j->max_len : 1));
  if (!s) return (void *)1;
  if (j->pairs) {
    for (int64_t i = j->tid; i < j->npairs; i += j->nthreads) {
      int64_t b = j->pairs[2 * i], h = j->pairs[2 * i + 1];
      attend_one(p, b, h, s, p->out + i * p->D, p->lse + i);
    }
  } else {
    const int64_t g = p->Hq / p->Hkv;
    for (int64_t u = j->tid; u < p->B * p->Hkv; u += j->nthreads) {
      int64_t b = u / p->Hkv, kh = u % p->Hkv;
      for (int64_t h = kh * g; h < (kh + 1) * g; ++h)
        attend_one(p, b, h, s, p->out + (b * p->Hq + h) * p->D, p->lse + b * p->Hq + h);
    }
  }
  free(s);
  return NULL;
}

static int run(const problem *p, const int32_t *pairs, int64_t npairs, int nthreads) {
  int64_t max_len = 0;
  for (int64_t b = 0; b < p->B; ++b)
    if (p->lens[b] > max_len) max_len = p->lens[b];
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  pthread_t th[512];
  job jobs[512];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].p = p;
    jobs[t].pairs = pairs;
    jobs[t].npairs = npairs;
    jobs[t].max_len = max_len;
    jobs[t].nthreads = nthreads;
    jobs[t].tid = t;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, worker, &jobs[t]);
  int rc = worker(&jobs[0]) != NULL;
  for (int t = 1; t < nthreads; ++t) {
    void *r = NULL;
    pthread_join(th[t], &r);
    rc |= r != NULL;
  }
  return rc;
}

static int fill(problem *p, const uint16_t *q, const int64_t *q_str, const void *k,
                const void *v, const int64_t *kv_str, const int32_t *tables,
                int64_t table_width, const int32_t *lens, int64_t B, int64_t Hq, int64_t Hkv,
                int64_t D, int64_t bs, double scale, int64_t window, const float *sinks, int64_t kv_fp8,
                double k_scale, double v_scale, double *out, double *lse) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0 || window < 0) return 2;
  if (kv_fp8 != 0 && kv_fp8 != 1) return 2;
  p->kv_fp8 = (int)kv_fp8;
  p->k_scale = k_scale;
  p->v_scale = v_scale;
  p->window = window;
  p->sinks = sinks;
  p->q = q;
  p->k = k;
  p->v = v;
  p->tables = tables;
  p->lens = lens;
  p->B = B;
  p->Hq = Hq;
  p->Hkv = Hkv;
  p->D = D;
  p->bs = bs;
  p->table_width = table_width;
  memcpy(p->q_str, q_str, sizeof(p->q_str));
  memcpy(p->kv_str, kv_str, sizeof(p->kv_str));
  p->scale = scale;
  p->out = out;
  p->lse = lse;
  return 0;
}

/* Every (b, h): out [B, Hq, D] and lse [B, Hq], double.  `window` 0 = every
 * token; `sinks` NULL = none; `kv_fp8` 0: k_cache/v_cache hold bf16 bits
 * (uint16), 1: E4M3 codes (uint8), dequantised with k_scale / v_scale (pass 1
 * for a bf16 cache).  Strides are in elements.  Returns 0 on success. */
int oracle_decode(const uint16_t *q, const int64_t *q_str, const void *k_cache, const void *v_cache,
                  const int64_t *kv_str, const int32_t *block_tables, int64_t table_width,
                  const int32_t *seq_lens, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t bs,
                  double scale, int64_t window, const float *sinks, int64_t kv_fp8, double k_scale,
                  double v_scale, double *out, double *lse, int nthreads) {
  problem p;
  int rc = fill(&p, q, q_str, k_cache, v_cache, kv_str, block_tables, table_width, seq_lens, B,
                Hq, Hkv, D, bs, scale, window, sinks, kv_fp8, k_scale, v_scale, out, lse);
  return rc ? rc : run(&p, NULL, 0, nthreads);
}

/* Selected (b, h) pairs only: out [npairs, D], lse [npairs]. */
int oracle_decode_pairs(const uint16_t *q, const int64_t *q_str, const void *k_cache,
                        const void *v_cache, const int64_t *kv_str, const int32_t *block_tables,
                        int64_t table_width, const int32_t *seq_lens, int64_t B, int64_t Hq,
                        int64_t Hkv, int64_t D, int64_t bs, double scale, int64_t window,
                        const float *sinks, int64_t kv_fp8, double k_scale, double v_scale,
                        const int32_t *pairs, int64_t npairs, double *out, double *lse, int nthreads) {
  problem p;
  int rc = fill(&p, q, q_str, k_cache, v_cache, kv_str, block_tables, table_width, seq_lens, B,
                Hq, Hkv, D, bs, scale, window, sinks, kv_fp8, k_scale, v_scale, out, lse);
  for (int64_t i = 0; !rc && i < npairs; ++i)
    if (pairs[2 * i] < 0 || pairs[2 * i] >= B || pairs[2 * i + 1] < 0 || pairs[2 * i + 1] >= Hq)
      rc = 2;
  return rc ? rc : run(&p, pairs, npairs, nthreads);
}
