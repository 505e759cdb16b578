/*
 * Seeded synthetic inputs for paged single-token decode attention.
 *
 * This module only draws numbers: it holds none of the attention arithmetic.
 * The GPU path and the CPU oracle both consume the bytes it produces, so the
 * two sides always see identical inputs.
 *
 * Generator: splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) used as a counter-based hash of
 * (seed, stream id, element index).  Every element is a pure function of
 * those three numbers, so any sub-range can be regenerated independently and
 * the fill is identical whatever the thread count.
 *
 *   uniform u in (0,1):  ((h >> 11) + 0.5) * 2^-53
 *   normal:              Box-Muller, sqrt(-2 ln u1) * cos(2 pi u2), with u1,u2
 *                        from the hashes of counters 2i and 2i+1
 *   bf16:                round-to-nearest-even of the fp32 value
 *   E4M3 codes:          the sample times a gain (1 / the tensor's scale),
 *                        rounded to nearest even onto the OCP FP8 E4M3 grid
 *                        (3 mantissa bits, exponent bias 7, subnormals below
 *                        2^-6), saturated at +-448, never NaN
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_DIST_NORMAL 0
#define SYNTH_DIST_UNIFORM_PM1 1

static inline uint64_t splitmix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return splitmix64(splitmix64(seed) ^ (stream * 0xD1B54A32D192ED03ull));
}

static inline uint64_t draw(uint64_t key, uint64_t counter) {
  return splitmix64(key + counter * 0x9E3779B97F4A7C15ull);
}

static inline double to_unit(uint64_t h) {
  return ((double)(h >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double sample(uint64_t key, uint64_t i, int dist) {
  if (dist == SYNTH_DIST_UNIFORM_PM1) return 2.0 * to_unit(draw(key, i)) - 1.0;
  double u1 = to_unit(draw(key, 2 * i));
  double u2 = to_unit(draw(key, 2 * i + 1));
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

static inline uint8_t f64_to_e4m3_rne(double x) {
  const uint8_t sign = signbit(x) ? 0x80 : 0;
  const double a = fabs(x);
  if (!(a > 0.0)) return sign;
  if (a >= 448.0) return sign | 0x7E;
  int e;
  frexp(a, &e);
  int E = e - 1; /* a in [2^E, 2^(E+1)) */
  if (E < -6) return sign | (uint8_t)nearbyint(a * 512.0); /* quantum 2^-9; 8 is the smallest normal */
  double m = nearbyint((a / ldexp(1.0, E) - 1.0) * 8.0);
  if (m == 8.0) {
    m = 0.0;
    E += 1;
  }
  if (E > 8 || (E == 8 && m > 6.0)) return sign | 0x7E;
  return sign | (uint8_t)(((E + 7) << 3) | (int)m);
}

/* ---- threaded driver ---------------------------------------------------- */

typedef struct {
  void *dst;             /* uint16 bf16 bits, or uint8 E4M3 codes when e4m3 */
  int e4m3;
  double gain;           /* E4M3 only: the sample is multiplied by it before rounding */
  const int64_t *blocks; /* NULL: dst is one flat range starting at counter `first` */
  int64_t nunits;        /* number of blocks, or number of elements when blocks==NULL */
  int64_t unit_elems;    /* elements per block (1 when blocks==NULL) */
  int64_t first;
  uint64_t key;
  int dist;
  int nthreads, tid;
} fill_job;

static inline void put(const fill_job *j, int64_t at, int64_t counter) {
  const double x = sample(j->key, (uint64_t)counter, j->dist);
  if (j->e4m3)
    ((uint8_t *)j->dst)[at] = f64_to_e4m3_rne(x * j->gain);
  else
    ((uint16_t *)j->dst)[at] = f32_to_bf16_rne((float)x);
}

static void *fill_worker(void *arg) {
  fill_job *j = (fill_job *)arg;
  int64_t lo = j->nunits * j->tid / j->nthreads;
  int64_t hi = j->nunits * (j->tid + 1) / j->nthreads;
  for (int64_t u = lo; u < hi; ++u) {
    if (j->blocks) {
      int64_t base = j->blocks[u] * j->unit_elems;
      for (int64_t e = 0; e < j->unit_elems; ++e) put(j, base + e, base + e);
    } else {
      put(j, u, j->first + u);
    }
  }
  return NULL;
}

static void run_fill(fill_job proto, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (proto.nunits < 4096) nthreads = 1;
  pthread_t th[256];
  fill_job jobs[256];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = proto;
    jobs[t].nthreads = nthreads;
    jobs[t].tid = t;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, fill_worker, &jobs[t]);
  fill_worker(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* Fill dst[0..n) with bf16 samples of counters first..first+n-1. */
void synth_fill_bf16(uint16_t *dst, int64_t n, int64_t first, uint64_t seed, uint64_t stream,
                     int dist, int nthreads) {
  fill_job j = {dst, 0, 1.0, NULL, n, 1, first, stream_key(seed, stream), dist, 1, 0};
  run_fill(j, nthreads);
}

/* For each listed block b, fill dst[b*block_elems .. (b+1)*block_elems) with the
 * samples of counters b*block_elems + e.  Unlisted blocks are not touched. */
void synth_fill_blocks_bf16(uint16_t *dst, const int64_t *blocks, int64_t nblocks,
                            int64_t block_elems, uint64_t seed, uint64_t stream, int dist,
                            int nthreads) {
  fill_job j = {dst, 0, 1.0, blocks, nblocks, block_elems, 0, stream_key(seed, stream), dist, 1, 0};
  run_fill(j, nthreads);
}

/* As synth_fill_blocks_bf16, with E4M3 codes of gain * sample (uint8). */
void synth_fill_blocks_e4m3(uint8_t *dst, const int64_t *blocks, int64_t nblocks,
                            int64_t block_elems, uint64_t seed, uint64_t stream, int dist,
                            double gain, int nthreads) {
  fill_job j = {dst, 1, gain, blocks, nblocks, block_elems, 0, stream_key(seed, stream), dist, 1, 0};
  run_fill(j, nthreads);
}

/* n uniforms in (0,1), in double. */
void synth_uniform_f64(double *dst, int64_t n, uint64_t seed, uint64_t stream) {
  uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) dst[i] = to_unit(draw(key, (uint64_t)i));
}

/* Uniform integer in [0, n) by Lemire's multiply-shift on a 64-bit draw. */
static inline int64_t below(uint64_t h, uint64_t n) {
  return (int64_t)(((unsigned __int128)h * n) >> 64);
}

/* The first k entries of a uniformly random permutation of 0..n-1
 * (Fisher-Yates, swap-from-the-front).  scratch must hold n int32. */
void synth_permutation_prefix(int32_t *dst, int32_t *scratch, int64_t n, int64_t k, uint64_t seed,
                              uint64_t stream) {
  uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) scratch[i] = (int32_t)i;
  if (k > n) k = n;
  for (int64_t i = 0; i < k; ++i) {
    int64_t j = i + below(draw(key, (uint64_t)i), (uint64_t)(n - i));
    int32_t t = scratch[i];
    scratch[i] = scratch[j];
    scratch[j] = t;
    dst[i] = scratch[i];
  }
}

/* Uniform integers in [lo, hi] inclusive. */
void synth_uniform_int(int32_t *dst, int64_t n, int32_t lo, int32_t hi, uint64_t seed,
                       uint64_t stream) {
  uint64_t key = stream_key(seed, stream);
  uint64_t span = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
  /* the offset is below 2^32; the sum, in [lo, hi], is formed in 64 bits */
  for (int64_t i = 0; i < n; ++i) dst[i] = (int32_t)((int64_t)lo + (int64_t)below(draw(key, (uint64_t)i), span));
}
