/* Sanitizer lane for the host side of libpad (the C ABI in include/pad.h).
 *
 * tests/test_host_sanitizers.py compiles the library's sources with the host
 * compiler under -fsanitize=address,undefined (device code unchanged) and links
 * this driver.  It runs on a machine without a GPU and never launches: it covers
 *   - pad_decode_plan / pad_decode_plan_ex over a grid of shapes, split
 *     requests and cache types (status in range; on success every plan field
 *     consistent with the shape), concurrently from several threads;
 *   - every decode entry point with host buffers and one argument broken at a
 *     time: an error status, a message from pad_last_error, and the output
 *     buffers byte-for-byte untouched (nothing is written before validation
 *     ends: "perf(rocke): prepare saved paged decode bindings once",
 *     rocm-libraries PR #13700, section "Testing Summary", poisons outputs and
 *     checks that the unused buffer stays untouched);
 *   - an empty batch (success, nothing launched), status strings, the ABI
 *     version, and the device-facing calls failing cleanly without a device.
 * Exit status 0 = clean.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pad.h"

static int failures = 0;
#define CHECK(cond, ...)                                   \
  do {                                                     \
    if (!(cond)) {                                         \
      fprintf(stderr, "FAIL %s:%d: ", __FILE__, __LINE__); \
      fprintf(stderr, __VA_ARGS__);                        \
      fputc('\n', stderr);                                 \
      ++failures;                                          \
    }                                                      \
  } while (0)

static int status_valid(pad_status st) { return st >= PAD_OK && st <= PAD_ERR_DEVICE_CHECK; }

static int has_message(void) {
  const char *m = pad_last_error();
  return m != NULL && m[0] != '\0';
}

/* ---- plans ------------------------------------------------------------- */

static void check_plan_fields(const pad_plan *p, int64_t B, int64_t Hq, int64_t Hkv, int64_t bs, int64_t mbps,
                              int32_t splits) {
  const int64_t g = Hq / Hkv, C = bs * mbps;
  CHECK(p->num_splits >= 1 && p->num_splits <= 256, "num_splits %d", p->num_splits);
  CHECK(p->partition_tokens >= 1 && p->partition_tokens % bs == 0, "partition_tokens %d (bs %lld)",
        p->partition_tokens, (long long)bs);
  CHECK(C == 0 || (int64_t)p->num_splits == (C + p->partition_tokens - 1) / p->partition_tokens || p->num_splits == 1,
        "num_splits %d != ceil(C / P) (C %lld, P %d)", p->num_splits, (long long)C, p->partition_tokens);
  CHECK(splits <= 0 || p->num_splits <= splits, "more partitions (%d) than requested (%d)", p->num_splits, splits);
  CHECK(p->heads_per_tile == 8 || p->heads_per_tile == 16 || p->heads_per_tile == 32, "heads_per_tile %d",
        p->heads_per_tile);
  CHECK((int64_t)p->head_tiles * p->heads_per_tile >= g && (int64_t)(p->head_tiles - 1) * p->heads_per_tile < g,
        "head_tiles %d x %d for group %lld", p->head_tiles, p->heads_per_tile, (long long)g);
  CHECK(p->warps_per_cta == 4 || p->warps_per_cta == 6, "warps_per_cta %d", p->warps_per_cta);
  CHECK(p->stage_tokens > 0 && p->stages >= 1 && p->stages <= 4, "stages %d x %d tokens", p->stages, p->stage_tokens);
  CHECK((int64_t)p->ctas == B * Hkv * p->head_tiles * (int64_t)p->num_splits, "ctas %d", p->ctas);
  CHECK(p->reduce == (p->num_splits > 1), "reduce %d with %d partitions", p->reduce, p->num_splits);
  CHECK(p->workspace_bytes >= 0 && p->control_bytes >= 0, "negative scratch sizes");
  CHECK(p->num_splits > 1 || (p->workspace_bytes == 0 && p->control_bytes == 0), "scratch without a merge");
  CHECK(p->num_splits == 1 || p->workspace_bytes >= (int64_t)B * Hq * p->num_splits * 4,
        "workspace %lld too small", (long long)p->workspace_bytes);
}

static void check_plans(void) {
  const int64_t Ds[] = {0, 32, 64, 96, 128, 256, 512};
  const int64_t heads[][2] = {{4, 1}, {32, 8}, {40, 8}, {32, 1}, {80, 2}, {16, 4}, {3, 2}, {0, 1}, {4, 0}, {64, 1}};
  const int64_t bss[] = {0, 1, 3, 4, 16, 32, 256, 512};
  const int64_t mbpss[] = {0, 1, 7, 4096, 1 << 20};
  const int32_t splitss[] = {-1, 0, 1, 3, 16, 256, 100000};
  const int32_t dtypes[] = {PAD_BF16, PAD_FP8_E4M3, PAD_F32, 99};
  long ok = 0, rejected = 0;
  for (size_t a = 0; a < sizeof(Ds) / sizeof(Ds[0]); ++a)
    for (size_t b = 0; b < sizeof(heads) / sizeof(heads[0]); ++b)
      for (size_t c = 0; c < sizeof(bss) / sizeof(bss[0]); ++c)
        for (size_t d = 0; d < sizeof(mbpss) / sizeof(mbpss[0]); ++d)
          for (size_t e = 0; e < sizeof(splitss) / sizeof(splitss[0]); ++e)
            for (size_t f = 0; f < sizeof(dtypes) / sizeof(dtypes[0]); ++f) {
              const int64_t B = 3, Hq = heads[b][0], Hkv = heads[b][1];
              pad_plan p;
              memset(&p, 0x5a, sizeof(p));
              pad_status st = pad_decode_plan_ex(B, Hq, Hkv, Ds[a], bss[c], mbpss[d], splitss[e], dtypes[f], 0, &p);
              CHECK(status_valid(st), "plan status %d", (int)st);
              if (st == PAD_OK) {
                ++ok;
                check_plan_fields(&p, B, Hq, Hkv, bss[c], mbpss[d], splitss[e]);
              } else {
                ++rejected;
                CHECK(has_message(), "plan rejected without a message");
              }
            }
  CHECK(ok > 100 && rejected > 100, "plan grid: %ld accepted, %ld rejected", ok, rejected);
  /* the bf16 entry equals the _ex entry with a bf16 cache */
  pad_plan a, b;
  memset(&a, 0, sizeof(a)); /* the struct has padding: compare what the calls write */
  memset(&b, 0, sizeof(b));
  CHECK(pad_decode_plan(32, 32, 8, 128, 16, 256, 0, 0, &a) == PAD_OK, "llama8b-shaped plan rejected");
  CHECK(pad_decode_plan_ex(32, 32, 8, 128, 16, 256, 0, PAD_BF16, 0, &b) == PAD_OK, "llama8b-shaped plan_ex rejected");
  CHECK(memcmp(&a, &b, sizeof(a)) == 0, "pad_decode_plan differs from pad_decode_plan_ex(bf16)");
  CHECK(pad_decode_plan(32, 32, 8, 128, 16, 256, 0, 0, NULL) != PAD_OK, "NULL plan accepted");
  CHECK(pad_decode_plan(-1, 32, 8, 128, 16, 256, 0, 0, &a) != PAD_OK, "negative batch accepted");
  CHECK(pad_decode_plan(32, 32, 8, 128, -16, 256, 0, 0, &a) != PAD_OK, "negative block size accepted");
  CHECK(pad_decode_plan(32, 32, 8, 128, 16, -1, 0, 0, &a) != PAD_OK, "negative table width accepted");
  /* sizes whose products would overflow 64 bits: rejected, not wrapped */
  const int64_t huge[][6] = {{(int64_t)1 << 62, 8, 8, 128, 16, 4},   {3, (int64_t)1 << 40, 1 << 20, 128, 16, 4},
                             {3, 32, 8, 128, 256, (int64_t)1 << 62}, {(int64_t)1 << 31, 2, 1, 64, 16, 4},
                             {1 << 20, 4096, 16, 128, 16, 4},         {3, 65537 * 2, 2, 128, 16, 4}};
  for (size_t i = 0; i < sizeof(huge) / sizeof(huge[0]); ++i) {
    pad_plan p;
    const int64_t *h = huge[i];
    CHECK(pad_decode_plan(h[0], h[1], h[2], h[3], h[4], h[5], 0, 0, &p) == PAD_ERR_UNSUPPORTED && has_message(),
          "oversized shape %zu not rejected", i);
  }
  /* the largest accepted sizes plan without overflow */
  CHECK(pad_decode_plan(1 << 20, 64, 1, 256, 256, 4096, 0, 0, &a) == PAD_OK && a.ctas > 0 && a.workspace_bytes > 0,
        "largest accepted shape did not plan");
}

static void *plan_thread(void *arg) {
  const int64_t t = (int64_t)(intptr_t)arg;
  for (int i = 0; i < 2000; ++i) {
    pad_plan p;
    const int64_t mbps = 1 + ((i * 37 + t * 11) % 3000);
    /* devices 1..8: the threads are the first to fill those slots of the
       library's per-device caches, at the same time */
    pad_status st = pad_decode_plan_ex(1 + (i % 64), 32, 1 + (i % 4 == 0 ? 0 : 7), 128, 16, mbps, i % 5,
                                       (i & 1) ? PAD_FP8_E4M3 : PAD_BF16, 1 + (i % 8), &p);
    if (st != PAD_OK && !has_message()) return (void *)1;
    if (i % 97 == 0) (void)pad_status_string(st);
  }
  return NULL;
}

static void check_plans_concurrently(void) {
  pthread_t th[4];
  for (intptr_t t = 0; t < 4; ++t) pthread_create(&th[t], NULL, plan_thread, (void *)t);
  for (int t = 0; t < 4; ++t) {
    void *r = NULL;
    pthread_join(th[t], &r);
    CHECK(r == NULL, "concurrent plan thread %d saw an error without a message", t);
  }
}

/* ---- decode entry points with host buffers ------------------------------ */

enum { B = 3, HQ = 8, HKV = 2, D = 128, BS = 16, NB = 12, MBPS = 4 };

typedef struct {
  pad_tensor q, k, v, tables, lens, out, lse, sinks;
  pad_decode_options opts;
  float scale;
  int32_t splits;
} call;

static uint16_t g_q[B * HQ * D], g_k[NB * HKV * BS * D], g_v[NB * HKV * BS * D];
static uint8_t g_k8[NB * HKV * BS * D], g_v8[NB * HKV * BS * D];
static int32_t g_tables[B * MBPS], g_lens[B];
static uint16_t g_out[B * HQ * D];
static float g_lse[B * HQ], g_sinks[HQ];
static unsigned char g_ws[1 << 16];

static pad_tensor tensor(void *data, int32_t dtype, int32_t ndim, const int64_t *shape) {
  pad_tensor t;
  memset(&t, 0, sizeof(t));
  t.data = data;
  t.dtype = dtype;
  t.ndim = ndim;
  int64_t s = 1;
  for (int i = ndim - 1; i >= 0; --i) {
    t.shape[i] = shape[i];
    t.stride[i] = s;
    s *= shape[i];
  }
  return t;
}

static call valid_call(void) {
  call c;
  memset(&c, 0, sizeof(c));
  const int64_t qs[3] = {B, HQ, D}, ks[4] = {NB, HKV, BS, D}, ts[2] = {B, MBPS}, ls[1] = {B}, es[2] = {B, HQ},
                ss[1] = {HQ};
  c.q = tensor(g_q, PAD_BF16, 3, qs);
  c.k = tensor(g_k, PAD_BF16, 4, ks);
  c.v = tensor(g_v, PAD_BF16, 4, ks);
  c.tables = tensor(g_tables, PAD_I32, 2, ts);
  c.lens = tensor(g_lens, PAD_I32, 1, ls);
  c.out = tensor(g_out, PAD_BF16, 3, qs);
  c.lse = tensor(g_lse, PAD_F32, 2, es);
  c.sinks = tensor(g_sinks, PAD_F32, 1, ss);
  c.opts.window_left = 0;
  c.opts.sinks = NULL;
  c.opts.k_scale = 0.f;
  c.opts.v_scale = 0.f;
  c.scale = 0.08838834764831845f;
  c.splits = 0;
  return c;
}

/* Every entry point on one call; each must fail and leave out / lse alone.
 * `expect_ok` marks calls that are valid without a device (an empty batch). */
static void run_all(call *c, const char *what, int expect_ok) {
  for (int entry = 0; entry < 6; ++entry) {
    memset(g_out, 0xA5, sizeof(g_out));
    memset(g_lse, 0xA5, sizeof(g_lse));
    pad_status st;
    switch (entry) {
      case 0:
        st = pad_decode(&c->q, &c->k, &c->v, &c->tables, &c->lens, c->scale, c->splits, &c->out, &c->lse, NULL);
        break;
      case 1:
        st = pad_decode_ex(&c->q, &c->k, &c->v, &c->tables, &c->lens, c->scale, c->splits, &c->opts, &c->out,
                           &c->lse, NULL);
        break;
      case 2:
        st = pad_decode_with_workspace(&c->q, &c->k, &c->v, &c->tables, &c->lens, c->scale, c->splits, &c->out,
                                       &c->lse, g_ws, sizeof(g_ws), NULL);
        break;
      case 3:
        st = pad_decode_with_workspace_ex(&c->q, &c->k, &c->v, &c->tables, &c->lens, c->scale, c->splits, &c->opts,
                                          &c->out, &c->lse, g_ws, sizeof(g_ws), NULL);
        break;
      case 4:
        st = pad_decode_static_scratch(&c->q, &c->k, &c->v, &c->tables, &c->lens, c->scale, c->splits, &c->out,
                                       &c->lse, NULL);
        break;
      default:
        st = pad_decode_tcgen05(&c->q, &c->k, &c->v, &c->tables, &c->lens, c->scale, c->splits, &c->out, &c->lse,
                                NULL);
        break;
    }
    CHECK(status_valid(st), "%s (entry %d): status %d out of range", what, entry, (int)st);
    if (expect_ok && entry != 5) {
      CHECK(st == PAD_OK, "%s (entry %d): status %d, want PAD_OK", what, entry, (int)st);
    } else if (!expect_ok) {
      CHECK(st != PAD_OK, "%s (entry %d): accepted", what, entry);
      CHECK(has_message(), "%s (entry %d): no message", what, entry);
    }
    unsigned char ref[sizeof(g_out)];
    memset(ref, 0xA5, sizeof(ref));
    CHECK(memcmp(g_out, ref, sizeof(g_out)) == 0, "%s (entry %d): out written", what, entry);
    CHECK(memcmp(g_lse, ref, sizeof(g_lse)) == 0, "%s (entry %d): lse written", what, entry);
  }
}

static void check_decode_validation(void) {
  call c;
  /* a well-formed call on host memory: rejected (no device / not device memory), nothing written */
  c = valid_call();
  run_all(&c, "valid shapes on host memory", 0);
  c = valid_call();
  c.k.dtype = c.v.dtype = PAD_FP8_E4M3;
  c.k.data = g_k8;
  c.v.data = g_v8;
  c.opts.k_scale = 0.5f;
  run_all(&c, "E4M3 cache on host memory", 0);
  /* an empty batch: valid everywhere but the tcgen05 entry is allowed either way */
  c = valid_call();
  c.q.shape[0] = c.out.shape[0] = c.tables.shape[0] = c.lens.shape[0] = c.lse.shape[0] = 0;
  run_all(&c, "empty batch", 1);

#define BROKEN(label, stmt) \
  do {                      \
    c = valid_call();       \
    stmt;                   \
    run_all(&c, label, 0);  \
  } while (0)
  BROKEN("q dtype f32", c.q.dtype = PAD_F32);
  BROKEN("q ndim 2", c.q.ndim = 2);
  BROKEN("q ndim 5", c.q.ndim = 5);
  BROKEN("unknown dtype", c.q.dtype = 77);
  BROKEN("k/v dtypes differ", c.v.dtype = PAD_FP8_E4M3);
  BROKEN("k dtype i32", c.k.dtype = PAD_I32);
  BROKEN("v shape differs", c.v.shape[1] = 1);
  BROKEN("head_dim mismatch", c.k.shape[3] = 64);
  BROKEN("group does not divide", (c.k.shape[1] = 3, c.v.shape[1] = 3));
  BROKEN("head_dim 96", (c.q.shape[2] = 96, c.k.shape[3] = c.v.shape[3] = 96, c.out.shape[2] = 96));
  BROKEN("block size 3", c.k.shape[2] = c.v.shape[2] = 3);
  BROKEN("block size 0", c.k.shape[2] = c.v.shape[2] = 0);
  BROKEN("no blocks", c.k.shape[0] = c.v.shape[0] = 0);
  BROKEN("tables rows", c.tables.shape[0] = B + 1);
  BROKEN("tables strided rows", c.tables.stride[1] = 2);
  BROKEN("tables dtype", c.tables.dtype = PAD_F32);
  BROKEN("lens count", c.lens.shape[0] = B - 1);
  BROKEN("lens strided", c.lens.stride[0] = 2);
  BROKEN("out shape", c.out.shape[1] = HQ - 1);
  BROKEN("out dtype", c.out.dtype = PAD_F32);
  BROKEN("lse shape", c.lse.shape[1] = HQ + 1);
  BROKEN("lse dtype", c.lse.dtype = PAD_BF16);
  BROKEN("q head_dim strided", c.q.stride[2] = 2);
  BROKEN("k head_dim strided", c.k.stride[3] = 2);
  BROKEN("q row misaligned", c.q.data = (char *)g_q + 2);
  BROKEN("k row misaligned", c.k.data = (char *)g_k + 8);
  BROKEN("lens misaligned", c.lens.data = (char *)g_lens + 2);
  BROKEN("negative stride", c.k.stride[0] = -c.k.stride[0]);
  BROKEN("negative shape", c.q.shape[1] = -8);
  BROKEN("NaN scale", c.scale = NAN);
  BROKEN("infinite scale", c.scale = INFINITY);
  BROKEN("negative splits", c.splits = -2);
  BROKEN("NULL q data", c.q.data = NULL);
  BROKEN("NULL out data", c.out.data = NULL);
  /* options (checked by the _ex entry points; the others ignore them) */
  c = valid_call();
  c.opts.window_left = -5;
  memset(g_out, 0, sizeof(g_out));
  CHECK(pad_decode_ex(&c.q, &c.k, &c.v, &c.tables, &c.lens, c.scale, 0, &c.opts, &c.out, &c.lse, NULL) != PAD_OK,
        "negative window accepted");
  c = valid_call();
  c.opts.k_scale = 2.f;
  CHECK(pad_decode_ex(&c.q, &c.k, &c.v, &c.tables, &c.lens, c.scale, 0, &c.opts, &c.out, &c.lse, NULL) != PAD_OK,
        "k_scale on a bf16 cache accepted");
  c = valid_call();
  c.k.dtype = c.v.dtype = PAD_FP8_E4M3;
  c.k.data = g_k8;
  c.v.data = g_v8;
  c.opts.v_scale = -1.f;
  CHECK(pad_decode_ex(&c.q, &c.k, &c.v, &c.tables, &c.lens, c.scale, 0, &c.opts, &c.out, &c.lse, NULL) != PAD_OK,
        "negative v_scale accepted");
  c.opts.v_scale = NAN;
  CHECK(pad_decode_ex(&c.q, &c.k, &c.v, &c.tables, &c.lens, c.scale, 0, &c.opts, &c.out, &c.lse, NULL) != PAD_OK,
        "NaN v_scale accepted");
  c = valid_call();
  c.sinks.shape[0] = HQ - 1;
  c.opts.sinks = &c.sinks;
  CHECK(pad_decode_ex(&c.q, &c.k, &c.v, &c.tables, &c.lens, c.scale, 0, &c.opts, &c.out, &c.lse, NULL) != PAD_OK,
        "sinks of the wrong length accepted");
  /* NULL descriptors */
  c = valid_call();
  CHECK(pad_decode(NULL, &c.k, &c.v, &c.tables, &c.lens, c.scale, 0, &c.out, &c.lse, NULL) != PAD_OK, "NULL q");
  CHECK(pad_decode(&c.q, NULL, &c.v, &c.tables, &c.lens, c.scale, 0, &c.out, &c.lse, NULL) != PAD_OK, "NULL k");
  CHECK(pad_decode(&c.q, &c.k, &c.v, NULL, &c.lens, c.scale, 0, &c.out, &c.lse, NULL) != PAD_OK, "NULL tables");
  CHECK(pad_decode(&c.q, &c.k, &c.v, &c.tables, NULL, c.scale, 0, &c.out, &c.lse, NULL) != PAD_OK, "NULL lens");
  CHECK(pad_decode(&c.q, &c.k, &c.v, &c.tables, &c.lens, c.scale, 0, NULL, &c.lse, NULL) != PAD_OK, "NULL out");
  CHECK(pad_decode_with_workspace(&c.q, &c.k, &c.v, &c.tables, &c.lens, c.scale, 4, &c.out, &c.lse, NULL, 1 << 20,
                                  NULL) != PAD_OK, "NULL workspace with a size accepted");
}

static void check_misc(void) {
  for (int s = -2; s <= 8; ++s) {
    const char *m = pad_status_string((pad_status)s);
    CHECK(m != NULL && m[0] != '\0', "no string for status %d", s);
  }
  CHECK(pad_abi_version() == PAD_ABI_VERSION, "ABI version %d, header %d", pad_abi_version(), PAD_ABI_VERSION);
  CHECK(pad_last_launch(NULL) != PAD_OK, "pad_last_launch(NULL) accepted");
  pad_launch_witness w;
  CHECK(status_valid(pad_last_launch(&w)), "pad_last_launch status out of range");
  uint32_t bits = 0;
  CHECK(status_valid(pad_check_device_errors(NULL, &bits)), "pad_check_device_errors status out of range");
  CHECK(status_valid(pad_release_workspace(0)), "pad_release_workspace(0) status out of range");
  CHECK(status_valid(pad_release_workspace(-1)), "pad_release_workspace(-1) status out of range");
}

int main(void) {
  check_misc();
  check_plans();
  check_plans_concurrently();
  check_decode_validation();
  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("host lane (C ABI): clean\n");
  return 0;
}
