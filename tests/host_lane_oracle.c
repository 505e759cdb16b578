/* Sanitizer lane for the CPU checker and the input generator.
 *
 * Built with -fsanitize=address,undefined by tests/test_host_sanitizers.py and
 * run on the CPU: every entry point of oracle/oracle.c and synth/synth.c on
 * small paged problems -- lengths 0, 1, one short of a page, a page, one past
 * it, the full table -- with and without window, sinks and an E4M3 cache, on
 * one and several threads.  Any out-of-bounds access, use of freed memory,
 * signed overflow or misaligned load aborts the run; the checks below add what
 * the sanitizers cannot see (finite results, -inf/zero for an empty sequence,
 * thread-count independence, valid permutations).  Exit status 0 = clean.
 *
 * Practice followed: the CPU lane that runs a project's host tests under the
 * address and undefined-behaviour sanitizers ("perf(BACKEND-ROCM): cooperate
 * across Q8_K activation blocks", vllm.cpp PR #2472, its CI classification
 * comment).  No GPU sanitizer is used.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

/* oracle/oracle.c */
int oracle_decode(const uint16_t *q, const int64_t *q_str, const void *k_cache, const void *v_cache,
                  const int64_t *kv_str, const int32_t *block_tables, int64_t table_width,
                  const int32_t *seq_lens, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t bs,
                  double scale, int64_t window, const float *sinks, int64_t kv_fp8, double k_scale,
                  double v_scale, double *out, double *lse, int nthreads);
int oracle_decode_pairs(const uint16_t *q, const int64_t *q_str, const void *k_cache,
                        const void *v_cache, const int64_t *kv_str, const int32_t *block_tables,
                        int64_t table_width, const int32_t *seq_lens, int64_t B, int64_t Hq,
                        int64_t Hkv, int64_t D, int64_t bs, double scale, int64_t window,
                        const float *sinks, int64_t kv_fp8, double k_scale, double v_scale,
                        const int32_t *pairs, int64_t npairs, double *out, double *lse, int nthreads);
/* synth/synth.c */
void synth_fill_bf16(uint16_t *dst, int64_t n, int64_t first, uint64_t seed, uint64_t stream, int dist,
                     int nthreads);
void synth_fill_blocks_bf16(uint16_t *dst, const int64_t *blocks, int64_t nblocks, int64_t block_elems,
                            uint64_t seed, uint64_t stream, int dist, int nthreads);
void synth_fill_blocks_e4m3(uint8_t *dst, const int64_t *blocks, int64_t nblocks, int64_t block_elems,
                            uint64_t seed, uint64_t stream, int dist, double gain, int nthreads);
void synth_uniform_f64(double *dst, int64_t n, uint64_t seed, uint64_t stream);
void synth_permutation_prefix(int32_t *dst, int32_t *scratch, int64_t n, int64_t k, uint64_t seed,
                              uint64_t stream);
void synth_uniform_int(int32_t *dst, int64_t n, int32_t lo, int32_t hi, uint64_t seed, uint64_t stream);

static int failures = 0;
#define CHECK(cond, ...)                      \
  do {                                        \
    if (!(cond)) {                            \
      fprintf(stderr, "FAIL %s:%d: ", __FILE__, __LINE__); \
      fprintf(stderr, __VA_ARGS__);           \
      fputc('\n', stderr);                    \
      ++failures;                             \
    }                                         \
  } while (0)

static void *xmalloc(size_t n) {
  void *p = malloc(n ? n : 1);
  if (!p) {
    fprintf(stderr, "out of memory\n");
    exit(2);
  }
  return p;
}

static void check_generator(void) {
  /* lengths around the single-thread cutoff and zero */
  const int64_t sizes[] = {0, 1, 7, 4095, 4096, 4097, 20000};
  for (size_t i = 0; i < sizeof(sizes) / sizeof(sizes[0]); ++i) {
    const int64_t n = sizes[i];
    uint16_t *a = xmalloc((size_t)n * 2), *b = xmalloc((size_t)n * 2);
    synth_fill_bf16(a, n, 3, 11, 2, 0, 1);
    synth_fill_bf16(b, n, 3, 11, 2, 0, 7);
    CHECK(n == 0 || memcmp(a, b, (size_t)n * 2) == 0, "bf16 fill depends on the thread count (n=%lld)", (long long)n);
    synth_fill_bf16(a, n, 0, 11, 2, 1, 300); /* above the thread cap */
    free(a);
    free(b);
  }
  /* block fills: scattered, in a pool larger than the blocks filled */
  const int64_t nb = 9, elems = 4096 + 3, pool = 16;
  int64_t blocks[9] = {15, 0, 7, 3, 12, 1, 9, 4, 10};
  uint16_t *kb = xmalloc((size_t)(pool * elems) * 2);
  uint8_t *k8 = xmalloc((size_t)(pool * elems));
  synth_fill_blocks_bf16(kb, blocks, nb, elems, 5, 1, 0, 4);
  synth_fill_blocks_e4m3(k8, blocks, nb, elems, 5, 1, 1, 0.5, 4);
  free(kb);
  free(k8);
  double u[257];
  synth_uniform_f64(u, 257, 1, 1);
  for (int i = 0; i < 257; ++i) CHECK(u[i] >= 0.0 && u[i] < 1.0, "uniform draw %g outside [0, 1)", u[i]);
  /* permutation prefixes: k < n, k == n, k > n, n == 1 */
  const int64_t ns[] = {1, 5, 64, 1000};
  for (size_t i = 0; i < sizeof(ns) / sizeof(ns[0]); ++i) {
    const int64_t n = ns[i];
    const int64_t ks[] = {0, 1, n / 2, n, n + 3};
    for (size_t j = 0; j < 5; ++j) {
      const int64_t k = ks[j], kk = k > n ? n : k;
      int32_t *dst = xmalloc((size_t)(kk + 1) * 4), *scratch = xmalloc((size_t)n * 4);
      char *seen = calloc((size_t)n, 1);
      synth_permutation_prefix(dst, scratch, n, k, 9, 4);
      for (int64_t t = 0; t < kk; ++t) {
        CHECK(dst[t] >= 0 && dst[t] < n, "permutation entry %d outside [0, %lld)", dst[t], (long long)n);
        if (dst[t] >= 0 && dst[t] < n) {
          CHECK(!seen[dst[t]], "permutation repeats %d", dst[t]);
          seen[dst[t]] = 1;
        }
      }
      free(dst);
      free(scratch);
      free(seen);
    }
  }
  int32_t ints[100];
  synth_uniform_int(ints, 100, -3, -3, 2, 2);
  for (int i = 0; i < 100; ++i) CHECK(ints[i] == -3, "uniform_int on one value gave %d", ints[i]);
  synth_uniform_int(ints, 100, -2147483647 - 1, 2147483647, 2, 3); /* the full int32 span */
  synth_uniform_int(ints, 100, 16, 32768, 2, 4);
  for (int i = 0; i < 100; ++i) CHECK(ints[i] >= 16 && ints[i] <= 32768, "uniform_int %d outside [16, 32768]", ints[i]);
}

/* One small paged problem through the oracle in every mode. */
static void check_oracle(int64_t Hq, int64_t Hkv, int64_t D, int64_t bs, int nhd) {
  const int64_t B = 7, width = 5, nblocks = B * width + 2;
  const int64_t cap = width * bs;
  const int32_t lens[7] = {0, 1, (int32_t)(bs > 1 ? bs - 1 : 1), (int32_t)bs, (int32_t)(bs + 1),
                           (int32_t)(cap - 1), (int32_t)cap};
  const int64_t kv_elems = nblocks * Hkv * bs * D;
  uint16_t *q = xmalloc((size_t)(B * Hq * D) * 2);
  uint16_t *k = xmalloc((size_t)kv_elems * 2), *v = xmalloc((size_t)kv_elems * 2);
  uint8_t *k8 = xmalloc((size_t)kv_elems), *v8 = xmalloc((size_t)kv_elems);
  synth_fill_bf16(q, B * Hq * D, 0, 1, 0, 0, 1);
  synth_fill_bf16(k, kv_elems, 0, 1, 1, 0, 2);
  synth_fill_bf16(v, kv_elems, 0, 1, 2, 1, 2);
  int64_t all[64];
  for (int64_t i = 0; i < nblocks; ++i) all[i] = i;
  synth_fill_blocks_e4m3(k8, all, nblocks, Hkv * bs * D, 1, 3, 0, 1.0, 2);
  synth_fill_blocks_e4m3(v8, all, nblocks, Hkv * bs * D, 1, 4, 0, 1.0, 2);
  int32_t *scratch = xmalloc((size_t)nblocks * 4), *tables = xmalloc((size_t)(B * width) * 4);
  synth_permutation_prefix(tables, scratch, nblocks, B * width, 3, 5);
  /* HND: [block, kv head, slot, d]; NHD: [block, slot, kv head, d] seen through strides */
  int64_t kv_str[4] = {Hkv * bs * D, bs * D, D, 1};
  if (nhd) {
    kv_str[1] = D;
    kv_str[2] = Hkv * D;
  }
  const int64_t q_str[3] = {Hq * D, D, 1};
  float *sinks = xmalloc((size_t)Hq * 4);
  for (int64_t h = 0; h < Hq; ++h) sinks[h] = (float)(0.25 * (double)h - 1.0);
  double *out = xmalloc((size_t)(B * Hq * D) * 8), *lse = xmalloc((size_t)(B * Hq) * 8);
  double *out3 = xmalloc((size_t)(B * Hq * D) * 8), *lse3 = xmalloc((size_t)(B * Hq) * 8);
  const double scale = 1.0 / sqrt((double)D);
  for (int fp8 = 0; fp8 <= 1; ++fp8) {
    const void *kc = fp8 ? (const void *)k8 : (const void *)k, *vc = fp8 ? (const void *)v8 : (const void *)v;
    const double ks = fp8 ? 0.046875 : 1.0, vs = fp8 ? 0.01953125 : 1.0;
    const int64_t windows[] = {0, 1, 3, cap + 7};
    for (int wi = 0; wi < 4; ++wi) {
      for (int with_sinks = 0; with_sinks <= 1; ++with_sinks) {
        const float *sk = with_sinks ? sinks : NULL;
        int rc = oracle_decode(q, q_str, kc, vc, kv_str, tables, width, lens, B, Hq, Hkv, D, bs, scale,
                               windows[wi], sk, fp8, ks, vs, out, lse, 1);
        CHECK(rc == 0, "oracle_decode rc %d", rc);
        rc = oracle_decode(q, q_str, kc, vc, kv_str, tables, width, lens, B, Hq, Hkv, D, bs, scale,
                           windows[wi], sk, fp8, ks, vs, out3, lse3, 3);
        CHECK(rc == 0, "oracle_decode (3 threads) rc %d", rc);
        CHECK(memcmp(out, out3, (size_t)(B * Hq * D) * 8) == 0 && memcmp(lse, lse3, (size_t)(B * Hq) * 8) == 0,
              "oracle result depends on the thread count");
        for (int64_t b = 0; b < B; ++b)
          for (int64_t h = 0; h < Hq; ++h) {
            const double l = lse[b * Hq + h];
            if (lens[b] == 0 && !with_sinks) {
              CHECK(isinf(l) && l < 0, "empty sequence: lse %g, want -inf", l);
            } else {
              CHECK(isfinite(l), "lse not finite (b=%lld h=%lld)", (long long)b, (long long)h);
            }
            for (int64_t d = 0; d < D; ++d) {
              const double o = out[(b * Hq + h) * D + d];
              CHECK(isfinite(o), "out not finite");
              if (lens[b] == 0) CHECK(o == 0.0, "empty sequence: out %g, want 0", o);
            }
          }
      }
    }
    /* selected pairs, including the first and the last */
    const int32_t pairs[6] = {0, 0, (int32_t)(B - 1), (int32_t)(Hq - 1), 3, (int32_t)(Hq / 2)};
    double pout[3 * 256], plse[3];
    int rc = oracle_decode_pairs(q, q_str, kc, vc, kv_str, tables, width, lens, B, Hq, Hkv, D, bs, scale, 0,
                                 NULL, fp8, ks, vs, pairs, 3, pout, plse, 2);
    CHECK(rc == 0, "oracle_decode_pairs rc %d", rc);
    rc = oracle_decode(q, q_str, kc, vc, kv_str, tables, width, lens, B, Hq, Hkv, D, bs, scale, 0, NULL, fp8,
                       ks, vs, out, lse, 1);
    for (int i = 0; i < 3; ++i) {
      const int64_t row = (int64_t)pairs[2 * i] * Hq + pairs[2 * i + 1];
      CHECK(memcmp(&pout[i * D], &out[row * D], (size_t)D * 8) == 0 && memcmp(&plse[i], &lse[row], 8) == 0,
            "pairs result differs from the full run");
    }
    /* rejected arguments: pair outside the batch, bad cache flag, head count */
    const int32_t bad[2] = {(int32_t)B, 0};
    CHECK(oracle_decode_pairs(q, q_str, kc, vc, kv_str, tables, width, lens, B, Hq, Hkv, D, bs, scale, 0, NULL,
                              fp8, ks, vs, bad, 1, pout, plse, 1) == 2, "pair outside the batch accepted");
    CHECK(oracle_decode(q, q_str, kc, vc, kv_str, tables, width, lens, B, Hq, Hkv, D, bs, scale, 0, NULL, 2, ks,
                        vs, out, lse, 1) == 2, "kv_fp8 = 2 accepted");
    CHECK(oracle_decode(q, q_str, kc, vc, kv_str, tables, width, lens, B, Hq, Hq + 1, D, bs, scale, 0, NULL,
                        fp8, ks, vs, out, lse, 1) == 2, "KV heads not dividing the query heads accepted");
    CHECK(oracle_decode(q, q_str, kc, vc, kv_str, tables, width, lens, B, Hq, Hkv, D, bs, scale, -1, NULL, fp8,
                        ks, vs, out, lse, 1) == 2, "negative window accepted");
  }
  /* an empty batch */
  CHECK(oracle_decode(q, q_str, k, v, kv_str, tables, width, lens, 0, Hq, Hkv, D, bs, scale, 0, NULL, 0, 1.0,
                      1.0, out, lse, 4) == 0, "empty batch rejected");
  free(q); free(k); free(v); free(k8); free(v8); free(scratch); free(tables); free(sinks);
  free(out); free(lse); free(out3); free(lse3);
}

int main(void) {
  check_generator();
  /* D 64/128/256, groups 1/4/5/32, page sizes 1/4/16/32, both cache layouts */
  check_oracle(4, 1, 128, 16, 0);
  check_oracle(8, 2, 64, 4, 1);
  check_oracle(5, 1, 256, 1, 0);
  check_oracle(32, 1, 128, 32, 1);
  check_oracle(10, 2, 64, 16, 0);
  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("host lane (oracle, input generator): clean\n");
  return 0;
}
