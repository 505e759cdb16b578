// Host side of libpad: argument validation, the per-shape launch plan, the
// split scratch and merge counters, and the launch.  Declared in include/pad.h.
#include "pad.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <map>
#include <set>
#include <mutex>
#include <string>
#include <utility>

#include "pad_internal.h"

namespace {

thread_local std::string g_last_error;
// pad_inject_stage_timeout: partition whose CTAs the next partition-kernel
// launch from this thread stalls (-1: none)
thread_local int32_t g_stall_partition = -1;

pad_status fail(pad_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

pad_status cuda_fail(cudaError_t e, const char *what) {
  return fail(PAD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

int ilog2(int64_t x) {
  int r = 0;
  while ((1ll << r) < x) ++r;
  return r;
}

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// ---- shape checks (no data access) ----------------------------------------

struct Shape {
  int64_t B, Hq, Hkv, D, bs, W, g;
  bool fp8;  // E4M3 cache
};

pad_status check_shape(const Shape &s, int32_t num_splits) {
  if (s.B < 0 || s.Hq <= 0 || s.Hkv <= 0 || s.D <= 0 || s.bs <= 0 || s.W <= 0)
    return fail(PAD_ERR_INVALID_ARG, "sizes must be positive (B >= 0): B=%lld Hq=%lld Hkv=%lld D=%lld bs=%lld W=%lld",
                (long long)s.B, (long long)s.Hq, (long long)s.Hkv, (long long)s.D, (long long)s.bs,
                (long long)s.W);
  if (s.Hq % s.Hkv != 0)
    return fail(PAD_ERR_INVALID_ARG, "num_q_heads (%lld) must be a multiple of num_kv_heads (%lld)",
                (long long)s.Hq, (long long)s.Hkv);
  if (num_splits < 0) return fail(PAD_ERR_INVALID_ARG, "num_splits must be >= 0 (got %d)", num_splits);
  if (s.D != 64 && s.D != 128 && s.D != 256)
    return fail(PAD_ERR_UNSUPPORTED, "head_dim %lld not supported (64, 128, 256)", (long long)s.D);
  if (!is_pow2(s.bs) || s.bs > 256)
    return fail(PAD_ERR_UNSUPPORTED, "block_size %lld must be a power of two in [1, 256]", (long long)s.bs);
  if (s.g > 256)
    return fail(PAD_ERR_UNSUPPORTED, "GQA group %lld exceeds 256 query heads per KV head", (long long)s.g);
  // Bounds that keep every product below (units, scratch bytes, row indices) in
  // range: sequences are indexed with 32-bit ints in the kernels, and (b, head)
  // rows of the split scratch number at most 2^31.
  if (s.B > 0x7fffffffll || s.Hq > 65536 || s.B * s.Hq > ((int64_t)1 << 31))
    return fail(PAD_ERR_UNSUPPORTED, "batch %lld x query heads %lld too large (at most 2^31 rows, 65536 heads)",
                (long long)s.B, (long long)s.Hq);
  if (s.W > ((int64_t)1 << 30) || s.W * s.bs > ((int64_t)1 << 30))
    return fail(PAD_ERR_UNSUPPORTED, "table capacity %lld blocks x %lld tokens too large (at most 2^30 tokens)",
                (long long)s.W, (long long)s.bs);
  return PAD_OK;
}

int sm_count(int device) {
  // per-device cache; threads that plan at once may both query and store the
  // same value, so the slots are atomic
  static std::atomic<int> cache[64];
  if (device < 0 || device >= 64) return 148;
  int n = cache[device].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cache[device].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Per-shape launch plan.  The lengths live on the device, so the plan sees only
// the table capacity C = W * bs.  Partitions are whole pages.  With num_splits==0
// the partition starts at max(512, 64 g) tokens, rounded up to a power of two
// (a unit's fixed cost -- start, merge of the four warps, partial and count --
// grows with the head group, so larger groups get longer partitions), and is
// halved, down to max(64, 16 g) (the split scratch a partition writes, g * D *
// 4 bytes, stays under 1/16 of the K/V bytes it streams, 4 * D * P), while the
// batch would give fewer than three units per SM of this device: a small batch
// still spreads over every SM.  Measured on B200 this picks the best of
// 64..8192-token partitions for the llama8b (512) and ragged_mqa (2048)
// batches, and for GQA batches of 1-16 sequences of 4096-8192 tokens the best
// or within 8% of it (fewer, longer units win there: each unit's start, the
// merge of its warps and its partial are fixed costs, and about three units
// per SM keep the SMs busy while leaving them few).  At most
// kMaxSplits partitions per sequence.  One CTA per unit; units past a
// sequence's length exit at once.
// PAD_LOG=1: one line on stderr for each distinct (shape, request, device,
// kernel) the library plans, the first time it plans it -- the launch geometry
// the decode entry points and pad_decode_plan choose.  Unset, empty or "0":
// silent.
// Any other value: one warning, then silent (a logging switch never fails a call).
bool plan_log_enabled() {
  static const bool on = [] {
    const char *v = getenv("PAD_LOG");
    if (v == nullptr || v[0] == '\0' || strcmp(v, "0") == 0) return false;
    if (strcmp(v, "1") == 0) return true;
    fprintf(stderr, "pad: PAD_LOG=%s ignored (0 or 1)\n", v);
    return false;
  }();
  return on;
}

void log_plan(const Shape &s, int32_t requested, int device, const pad_plan &p, bool umma) {
  if (!plan_log_enabled()) return;
  char line[512];
  snprintf(line, sizeof line,
           "pad: plan B=%lld Hq=%lld Hkv=%lld D=%lld bs=%lld capacity=%lld kv=%s num_splits=%d device=%d -> "
           "kernel=%s S=%d P=%d heads_per_tile=%d head_tiles=%d stages=%dx%d warps=%d ctas=%d ctas_per_sm=%d "
           "workspace_bytes=%lld control_bytes=%lld\n",
           (long long)s.B, (long long)s.Hq, (long long)s.Hkv, (long long)s.D, (long long)s.bs,
           (long long)(s.W * s.bs), s.fp8 ? "e4m3" : "bf16", requested, device, umma ? "tcgen05" : "partition",
           p.num_splits, p.partition_tokens, p.heads_per_tile, p.head_tiles, p.stages, p.stage_tokens,
           p.warps_per_cta, p.ctas, p.ctas_per_sm, (long long)p.workspace_bytes, (long long)p.control_bytes);
  static std::mutex mu;
  static std::set<std::string> seen;
  std::lock_guard<std::mutex> lock(mu);
  if (seen.insert(line).second) fputs(line, stderr);
}

constexpr int kSplitUnitsPerSm = 3;  // the automatic split halves P until the launch has this many units per SM

void make_plan(const Shape &s, int32_t num_splits, int device, pad_plan *plan, bool tcgen05 = false) {
  const int64_t C = s.W * s.bs;
  int hpt = s.g <= 8 ? 8 : (s.g <= 16 ? 16 : 32);
  if (hpt > pad::max_heads_per_tile((int)s.D)) hpt = pad::max_heads_per_tile((int)s.D);
  const int64_t HT = (s.g + hpt - 1) / hpt;
  int64_t P;
  if (num_splits >= 1) {
    P = round_up((C + num_splits - 1) / num_splits, s.bs);
  } else {
    const int64_t p_floor = round_up(16 * s.g > 64 ? 16 * s.g : 64, 64);
    P = 512;
    while (P < 64 * s.g) P *= 2;
    const int64_t min_units = (int64_t)kSplitUnitsPerSm * sm_count(device < 0 ? 0 : device);
    const int64_t pairs = s.B * s.Hkv * HT;
    while (P / 2 >= p_floor && P / 2 >= s.bs && pairs * ((C + P - 1) / P) < min_units) P /= 2;
    P = round_up(P, s.bs);
  }
  if (P > round_up(C, s.bs)) P = round_up(C, s.bs);
  if (P < s.bs) P = s.bs;
  if ((C + P - 1) / P > pad::kMaxSplits) P = round_up((C + pad::kMaxSplits - 1) / pad::kMaxSplits, s.bs);
  const int64_t S = (C + P - 1) / P;
  const int64_t units = s.B * s.Hkv * HT * S;
  plan->num_splits = (int32_t)S;
  plan->partition_tokens = (int32_t)P;
  plan->heads_per_tile = hpt;
  plan->head_tiles = (int32_t)HT;
  const bool umma = tcgen05 && !s.fp8 && pad::umma_eligible((int)s.D, hpt, (int)s.bs);
  plan->warps_per_cta = umma ? pad::kUmmaWarps : pad::warps_for((int)s.D, hpt, s.fp8);
  plan->stage_tokens = umma ? pad::kUmmaStageTokens : pad::stage_tokens_for((int)s.D, hpt, s.fp8);
  plan->stages = umma ? pad::umma_stages() : pad::partition_stages((int)s.D, hpt, s.fp8);
  // one CTA per unit (both kernels)
  plan->ctas = (int32_t)(units > 0x7fffffffll ? 0x7fffffffll : units);
  plan->ctas_per_sm = umma ? pad::kUmmaCtasPerSm
                           : pad::ctas_per_sm_choice((int)s.D, hpt, s.fp8, units, sm_count(device < 0 ? 0 : device));
  plan->reduce = S > 1 ? 1 : 0;
  plan->workspace_bytes =
      (int64_t)pad::workspace_layout(s.B, s.Hq, S, s.D, units, pad::schedules_units(s.B, S, P, hpt)).total;
  plan->control_bytes = (int64_t)pad::control_layout(s.B, s.Hkv, HT, S).total;
  log_plan(s, num_splits, device, *plan, umma);
}

// ---- TMA tensor maps of the K/V caches --------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda); null if the driver does not provide it.
EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
    else
      cudaGetLastError();
  });
  return fn;
}

// A [num_blocks, Hkv, bs, D] bf16 cache as the 5-D tensor (64 head_dim
// elements, slot, head_dim / 64, kv head, block) with boxes of (64, box_rows,
// D / 64, 1, 1) and the 128-byte swizzle.  Byte strides of size-1 dimensions
// are never used; a natural value stands in for them.
pad_status encode_cache_map(CUtensorMap *map, const pad_tensor *t, int box_rows_, const char *name) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return fail(PAD_ERR_CUDA, "the CUDA driver does not provide cuTensorMapEncodeTiled");
  const int64_t NB = t->shape[0], Hkv = t->shape[1], bs = t->shape[2], D = t->shape[3];
  const bool fp8 = t->dtype == PAD_FP8_E4M3;
  const int64_t eb = fp8 ? 1 : 2;                 // bytes per element
  const int64_t rowb = D * eb, rw = rowb < 128 ? rowb : 128;  // row bytes; bytes per column block
  auto stride_bytes = [&](int i, int64_t natural) -> cuuint64_t {
    return (cuuint64_t)(t->shape[i] > 1 ? t->stride[i] * eb : natural);
  };
  const cuuint64_t dims[5] = {(cuuint64_t)(rw / eb), (cuuint64_t)bs, (cuuint64_t)(rowb / rw), (cuuint64_t)Hkv,
                              (cuuint64_t)NB};
  const cuuint64_t strides[4] = {stride_bytes(2, rowb), (cuuint64_t)rw, stride_bytes(1, bs * rowb),
                                 stride_bytes(0, Hkv * bs * rowb)};
  const cuuint32_t box[5] = {(cuuint32_t)(rw / eb), (cuuint32_t)box_rows_, (cuuint32_t)(rowb / rw), 1, 1};
  const cuuint32_t elem[5] = {1, 1, 1, 1, 1};
  const CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, t->data,
                         dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         rw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(PAD_ERR_INVALID_ARG, "%s: strides/shape not expressible as a TMA tensor (cuTensorMapEncodeTiled %d)",
                name, (int)r);
  return PAD_OK;
}

// q [B, Hq, D] as the 4-D tensor (64 head_dim elements, head, head_dim / 64, b)
// with boxes of (64, heads, D / 64, 1) and the 128-byte swizzle.
pad_status encode_q_map(CUtensorMap *map, const pad_tensor *q, int heads) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return fail(PAD_ERR_CUDA, "the CUDA driver does not provide cuTensorMapEncodeTiled");
  const int64_t B = q->shape[0], Hq = q->shape[1], D = q->shape[2];
  const cuuint64_t dims[4] = {64, (cuuint64_t)Hq, (cuuint64_t)(D / 64), (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)(Hq > 1 ? q->stride[1] * 2 : D * 2), 128,
                                 (cuuint64_t)(B > 1 ? q->stride[0] * 2 : Hq * D * 2)};
  const cuuint32_t box[4] = {64, (cuuint32_t)heads, (cuuint32_t)(D / 64), 1};
  const cuuint32_t elem[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, q->data, dims, strides, box, elem,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PAD_ERR_INVALID_ARG, "q: strides/shape not expressible as a TMA tensor (%d)", (int)r);
  return PAD_OK;
}

// ---- tensor descriptor checks -----------------------------------------------

pad_status check_tensor(const pad_tensor *t, const char *name, pad_dtype dt, int ndim) {
  if (t == nullptr) return fail(PAD_ERR_INVALID_ARG, "%s is NULL", name);
  if (t->data == nullptr) return fail(PAD_ERR_INVALID_ARG, "%s.data is NULL", name);
  if (t->dtype != dt) return fail(PAD_ERR_INVALID_ARG, "%s has dtype %d, expected %d", name, t->dtype, (int)dt);
  if (t->ndim != ndim) return fail(PAD_ERR_INVALID_ARG, "%s has %d dims, expected %d", name, t->ndim, ndim);
  for (int i = 0; i < ndim; ++i) {
    if (t->shape[i] < 0) return fail(PAD_ERR_INVALID_ARG, "%s.shape[%d] < 0", name, i);
    if (t->stride[i] < 0) return fail(PAD_ERR_INVALID_ARG, "%s.stride[%d] < 0", name, i);
  }
  return PAD_OK;
}

// rows of `elem_bytes`-byte elements along the last dim must be contiguous and 16-byte aligned
pad_status check_rows16(const pad_tensor *t, const char *name, int64_t elem_bytes = 2) {
  const int last = t->ndim - 1;
  if (t->stride[last] != 1) return fail(PAD_ERR_INVALID_ARG, "%s: last dim must be contiguous", name);
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0)
    return fail(PAD_ERR_INVALID_ARG, "%s: data must be 16-byte aligned", name);
  for (int i = 0; i < last; ++i)
    if ((t->stride[i] * elem_bytes) % 16 != 0 && t->shape[i] > 1)
      return fail(PAD_ERR_INVALID_ARG, "%s: stride[%d]=%lld is not a multiple of 16 bytes", name, i,
                  (long long)t->stride[i]);
  return PAD_OK;
}

pad_status check_device_ptr(const void *p, int device, const char *name) {
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(PAD_ERR_INVALID_ARG, "%s: not a CUDA pointer (%s)", name, cudaGetErrorString(e));
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(PAD_ERR_INVALID_ARG, "%s: must be device memory", name);
  if (a.type == cudaMemoryTypeDevice && a.device != device)
    return fail(PAD_ERR_INVALID_ARG, "%s: lives on device %d, current device is %d", name, a.device, device);
  return PAD_OK;
}

// ---- library-owned buffers, one of each kind per (device, stream) -----------
//
// Partials: split outputs, no initial contents needed.  Control: merge
// counters, zero-filled when (re)allocated and left zero by every launch that
// completes, so one buffer serves calls of any shape in stream order.

struct Workspace {
  void *ptr = nullptr;
  size_t bytes = 0;
};
std::mutex g_ws_mu;
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;   // partials
std::map<std::pair<int, cudaStream_t>, Workspace> g_ctl;  // control blocks

pad_status get_buffer(std::map<std::pair<int, cudaStream_t>, Workspace> &pool, int device, cudaStream_t stream,
                      size_t bytes, void **out) {
  std::lock_guard<std::mutex> lock(g_ws_mu);
  Workspace &w = pool[{device, stream}];
  if (w.bytes >= bytes) {
    *out = w.ptr;
    return PAD_OK;
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(stream, &cs);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
  if (cs != cudaStreamCaptureStatusNone)
    return fail(PAD_ERR_WORKSPACE,
                "split scratch must grow to %zu bytes while the stream is being captured; "
                "run one call with this shape outside capture first", bytes);
  if (w.ptr != nullptr) {
    // queued work on this stream may still use the old buffer
    e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    cudaFree(w.ptr);
    w.ptr = nullptr;
    w.bytes = 0;
  }
  size_t want = bytes + bytes / 4;  // headroom for nearby shapes
  e = cudaMalloc(&w.ptr, want);
  if (e != cudaSuccess) {
    cudaGetLastError();
    e = cudaMalloc(&w.ptr, bytes);
    want = bytes;
  }
  if (e != cudaSuccess) {
    w.ptr = nullptr;
    return fail(PAD_ERR_WORKSPACE, "cudaMalloc(%zu) for split scratch failed: %s", bytes, cudaGetErrorString(e));
  }
  e = cudaMemsetAsync(w.ptr, 0, want, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(library scratch)");
  w.bytes = want;
  *out = w.ptr;
  return PAD_OK;
}

// ---- one call: validate, plan, bind, launch ---------------------------------

struct Prepared {
  pad::PartitionParams p;
  pad_plan plan;
  bool umma;  // the tcgen05 kernel runs this shape
  pad::WorkspaceLayout ws;
  pad::ControlLayout cl;
  int D;
  int device;
  bool kv_fp8;
  bool ordered;  // the launch orders its units (schedule pass first)
};

pad_status prepare(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                   const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale, int32_t num_splits,
                   const pad_tensor *out, const pad_tensor *lse, Prepared *pr, bool *empty,
                   bool tcgen05 = false, const pad_decode_options *opts = nullptr) {
  pad_status st;
  *empty = false;
  if ((st = check_tensor(q, "q", PAD_BF16, 3)) != PAD_OK) return st;
  // the cache is bf16 or E4M3, K and V alike
  const bool fp8 = k_cache != nullptr && k_cache->dtype == PAD_FP8_E4M3;
  const pad_dtype kv_dt = fp8 ? PAD_FP8_E4M3 : PAD_BF16;
  if ((st = check_tensor(k_cache, "k_cache", kv_dt, 4)) != PAD_OK) return st;
  if ((st = check_tensor(v_cache, "v_cache", kv_dt, 4)) != PAD_OK) return st;
  if ((st = check_tensor(block_tables, "block_tables", PAD_I32, 2)) != PAD_OK) return st;
  if ((st = check_tensor(seq_lens, "seq_lens", PAD_I32, 1)) != PAD_OK) return st;
  if ((st = check_tensor(out, "out", PAD_BF16, 3)) != PAD_OK) return st;
  if (lse != nullptr && (st = check_tensor(lse, "lse", PAD_F32, 2)) != PAD_OK) return st;

  const int64_t B = q->shape[0], Hq = q->shape[1], D = q->shape[2];
  const int64_t NB = k_cache->shape[0], Hkv = k_cache->shape[1], bs = k_cache->shape[2];
  for (int i = 0; i < 4; ++i)
    if (v_cache->shape[i] != k_cache->shape[i])
      return fail(PAD_ERR_INVALID_ARG, "v_cache.shape[%d]=%lld differs from k_cache", i, (long long)v_cache->shape[i]);
  if (k_cache->shape[3] != D)
    return fail(PAD_ERR_INVALID_ARG, "k_cache head_dim %lld != q head_dim %lld", (long long)k_cache->shape[3], (long long)D);
  if (block_tables->shape[0] != B)
    return fail(PAD_ERR_INVALID_ARG, "block_tables has %lld rows, batch is %lld", (long long)block_tables->shape[0], (long long)B);
  if (block_tables->stride[1] != 1 && block_tables->shape[1] > 1)
    return fail(PAD_ERR_INVALID_ARG, "block_tables rows must be contiguous");
  if (seq_lens->shape[0] != B)
    return fail(PAD_ERR_INVALID_ARG, "seq_lens has %lld entries, batch is %lld", (long long)seq_lens->shape[0], (long long)B);
  if (seq_lens->stride[0] != 1 && B > 1) return fail(PAD_ERR_INVALID_ARG, "seq_lens must be contiguous");
  if (out->shape[0] != B || out->shape[1] != Hq || out->shape[2] != D)
    return fail(PAD_ERR_INVALID_ARG, "out shape must equal q shape [%lld, %lld, %lld]", (long long)B, (long long)Hq, (long long)D);
  if (lse != nullptr && (lse->shape[0] != B || lse->shape[1] != Hq))
    return fail(PAD_ERR_INVALID_ARG, "lse shape must be [B, Hq] = [%lld, %lld]", (long long)B, (long long)Hq);
  if (!isfinite(scale)) return fail(PAD_ERR_INVALID_ARG, "scale must be finite");
  if (NB <= 0 || NB > 0x7fffffffll) return fail(PAD_ERR_INVALID_ARG, "num_blocks %lld out of range", (long long)NB);
  if ((st = check_rows16(q, "q")) != PAD_OK) return st;
  if ((st = check_rows16(k_cache, "k_cache", fp8 ? 1 : 2)) != PAD_OK) return st;
  if ((st = check_rows16(v_cache, "v_cache", fp8 ? 1 : 2)) != PAD_OK) return st;
  if ((st = check_rows16(out, "out")) != PAD_OK) return st;
  if (reinterpret_cast<uintptr_t>(block_tables->data) % 4 || reinterpret_cast<uintptr_t>(seq_lens->data) % 4 ||
      (lse != nullptr && reinterpret_cast<uintptr_t>(lse->data) % 4))
    return fail(PAD_ERR_INVALID_ARG, "int32/fp32 tensors must be 4-byte aligned");

  Shape s{B, Hq, Hkv, D, bs, block_tables->shape[1], Hkv > 0 ? Hq / Hkv : 0, fp8};
  if ((st = check_shape(s, num_splits)) != PAD_OK) return st;
  // dequantisation scales: 0 reads as 1; an E4M3 cache takes any finite
  // positive value, a bf16 cache only 1
  float k_scale = 1.f, v_scale = 1.f;
  if (opts != nullptr) {
    k_scale = opts->k_scale == 0.f ? 1.f : opts->k_scale;
    v_scale = opts->v_scale == 0.f ? 1.f : opts->v_scale;
    if (!(isfinite(k_scale) && k_scale > 0.f) || !(isfinite(v_scale) && v_scale > 0.f))
      return fail(PAD_ERR_INVALID_ARG, "k_scale and v_scale must be finite and positive (or 0 for 1)");
    if (!fp8 && (k_scale != 1.f || v_scale != 1.f))
      return fail(PAD_ERR_INVALID_ARG, "k_scale / v_scale apply to an E4M3 cache only (bf16 cache: 0 or 1)");
  }
  if (B == 0) {
    *empty = true;
    return PAD_OK;
  }

  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if ((st = check_device_ptr(q->data, device, "q")) != PAD_OK) return st;
  if ((st = check_device_ptr(k_cache->data, device, "k_cache")) != PAD_OK) return st;
  if ((st = check_device_ptr(v_cache->data, device, "v_cache")) != PAD_OK) return st;
  if ((st = check_device_ptr(block_tables->data, device, "block_tables")) != PAD_OK) return st;
  if ((st = check_device_ptr(seq_lens->data, device, "seq_lens")) != PAD_OK) return st;
  if ((st = check_device_ptr(out->data, device, "out")) != PAD_OK) return st;
  if (lse != nullptr && (st = check_device_ptr(lse->data, device, "lse")) != PAD_OK) return st;

  if (tcgen05 && (fp8 || !pad::umma_eligible((int)D, s.g <= 8 ? 8 : (s.g <= 16 ? 16 : 32), (int)bs)))
    return fail(PAD_ERR_UNSUPPORTED,
                "the tcgen05 kernel takes a bf16 cache with groups of 17..32 query heads per KV head at head_dim "
                "128 and a block size of at least 8 (got %s, group %lld, head_dim %lld, block size %lld)",
                fp8 ? "E4M3" : "bf16", (long long)s.g, (long long)D, (long long)bs);
  make_plan(s, num_splits, device, &pr->plan, tcgen05);
  const int64_t units = B * Hkv * pr->plan.head_tiles * (int64_t)pr->plan.num_splits;
  if (units > 0x7fffffffll) return fail(PAD_ERR_UNSUPPORTED, "too many work units (%lld) for one launch", (long long)units);
  pr->ordered = pad::schedules_units(B, pr->plan.num_splits, pr->plan.partition_tokens, pr->plan.heads_per_tile);
  pr->ws = pad::workspace_layout(B, Hq, pr->plan.num_splits, D, units, pr->ordered);
  pr->cl = pad::control_layout(B, Hkv, pr->plan.head_tiles, pr->plan.num_splits);

  uint32_t *err = nullptr;
  if ((e = pad::device_error_word(device, &err)) != cudaSuccess) return cuda_fail(e, "error word");

  pad::PartitionParams &p = pr->p;
  p = pad::PartitionParams{};
  pr->umma = tcgen05;
  const int rows = pr->umma ? 8 : pad::box_rows((int)bs, (int)D, pr->plan.heads_per_tile, fp8);
  if ((st = encode_cache_map(&p.tmk, k_cache, rows, "k_cache")) != PAD_OK) return st;
  if ((st = encode_cache_map(&p.tmv, v_cache, rows, "v_cache")) != PAD_OK) return st;
  if (pr->umma && (st = encode_q_map(&p.tmq, q, pr->plan.heads_per_tile)) != PAD_OK) return st;
  p.q = static_cast<const uint16_t *>(q->data);
  p.q_sb = q->stride[0];
  p.q_sh = q->stride[1];
  p.k = static_cast<const uint16_t *>(k_cache->data);
  p.v = static_cast<const uint16_t *>(v_cache->data);
  p.k_sblk = k_cache->stride[0];
  p.k_sh = k_cache->stride[1];
  p.k_ss = k_cache->stride[2];
  p.v_sblk = v_cache->stride[0];
  p.v_sh = v_cache->stride[1];
  p.v_ss = v_cache->stride[2];
  p.tables = static_cast<const int32_t *>(block_tables->data);
  p.table_stride = block_tables->stride[0];
  p.max_blocks = (int32_t)block_tables->shape[1];
  p.num_blocks = (int32_t)NB;
  p.seq_lens = static_cast<const int32_t *>(seq_lens->data);
  p.B = (int32_t)B;
  p.Hq = (int32_t)Hq;
  p.Hkv = (int32_t)Hkv;
  p.g = (int32_t)(Hq / Hkv);
  p.HT = pr->plan.head_tiles;
  p.bs_log2 = ilog2(bs);
  p.P = pr->plan.partition_tokens;
  p.S = pr->plan.num_splits;
  p.n_units = (uint32_t)units;
  p.scale_log2 = (float)((double)scale * (double)k_scale * 1.4426950408889634);
  p.v_scale = v_scale;
  if (opts != nullptr) {
    if (opts->window_left < 0) return fail(PAD_ERR_INVALID_ARG, "window_left must be >= 0 (got %d)", opts->window_left);
    p.window = opts->window_left;
    if (opts->sinks != nullptr) {
      const pad_tensor *sk = opts->sinks;
      if ((st = check_tensor(sk, "sinks", PAD_F32, 1)) != PAD_OK) return st;
      if (sk->shape[0] != Hq) return fail(PAD_ERR_INVALID_ARG, "sinks must be fp32 [Hq] = [%lld]", (long long)Hq);
      if (sk->stride[0] != 1 && Hq > 1) return fail(PAD_ERR_INVALID_ARG, "sinks must be contiguous");
      if (reinterpret_cast<uintptr_t>(sk->data) % 4) return fail(PAD_ERR_INVALID_ARG, "sinks must be 4-byte aligned");
      if ((st = check_device_ptr(sk->data, device, "sinks")) != PAD_OK) return st;
      p.sinks = static_cast<const float *>(sk->data);
    }
  }
  p.out = static_cast<uint16_t *>(out->data);
  p.o_sb = out->stride[0];
  p.o_sh = out->stride[1];
  p.lse = lse != nullptr ? static_cast<float *>(lse->data) : nullptr;
  p.lse_sb = lse != nullptr ? lse->stride[0] : 0;
  p.lse_sh = lse != nullptr ? lse->stride[1] : 0;
  p.err = err;
  p.stall_partition = tcgen05 ? -1 : g_stall_partition;
  if ((e = pad::device_witness(device, &p.witness)) != cudaSuccess) return cuda_fail(e, "launch witness");
  pr->D = (int)D;
  pr->device = device;
  pr->kv_fp8 = fp8;
  return PAD_OK;
}

void bind_buffers(Prepared &pr, void *partials, void *control) {
  // No partials buffer (one partition per sequence, nothing to merge): the
  // kernel never reads these, and no offset is applied to a null pointer.
  char *base = static_cast<char *>(partials);
  pr.p.o_part = base != nullptr ? reinterpret_cast<float *>(base + pr.ws.o_part) : nullptr;
  pr.p.lse_part = base != nullptr ? reinterpret_cast<float *>(base + pr.ws.lse_part) : nullptr;
  pr.p.order = base != nullptr && pr.ordered ? reinterpret_cast<uint32_t *>(base + pr.ws.order) : nullptr;
  pr.p.counters = pr.cl.total > 0 ? reinterpret_cast<uint32_t *>(static_cast<char *>(control) + pr.cl.counters)
                                  : nullptr;
}

pad_status check_caller_buffer(const Prepared &pr, void *buf, size_t bytes, size_t need, const char *name) {
  if (need == 0) return PAD_OK;
  if (buf == nullptr) return fail(PAD_ERR_INVALID_ARG, "%s is NULL but %zu bytes are needed", name, need);
  if (bytes < need) return fail(PAD_ERR_INVALID_ARG, "%s has %zu bytes, %zu needed", name, bytes, need);
  if (reinterpret_cast<uintptr_t>(buf) % 256 != 0) return fail(PAD_ERR_INVALID_ARG, "%s must be 256-byte aligned", name);
  return check_device_ptr(buf, pr.device, name);
}

pad_status run(const Prepared &pr, cudaStream_t stream) {
  cudaError_t e = pr.p.order != nullptr ? pad::launch_schedule(pr.p, stream) : cudaSuccess;
  if (e != cudaSuccess) return cuda_fail(e, "unit schedule launch");
  e = pr.umma ? pad::launch_umma(pr.p, pr.plan.ctas, stream)
              : pad::launch_partition(pr.p, pr.D, pr.plan.heads_per_tile, pr.kv_fp8, pr.plan.ctas,
                                      pr.plan.ctas_per_sm, stream);
  if (!pr.umma) g_stall_partition = -1;  // the test hook is one-shot
  return e == cudaSuccess ? PAD_OK : cuda_fail(e, "partition kernel launch");
}

}  // namespace

namespace pad {
// Lets other translation units of the library report a failure through
// pad_last_error().
void set_last_error(const char *msg) { g_last_error = msg; }

pad_status decode_with_scratch_array(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                                     const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                                     int32_t num_splits, pad_tensor *out, pad_tensor *lse,
                                     pad_status (*scratch_address)(void **), size_t scratch_bytes,
                                     cudaStream_t stream) {
  Prepared pr;
  bool empty = false;
  pad_status st = prepare(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits, out, lse, &pr, &empty);
  if (st != PAD_OK || empty) return st;
  // the control block sits at the array's start, the partials after it (the
  // control block's size is a multiple of 256 bytes, so they stay aligned)
  const size_t need = pr.cl.total + pr.ws.total;
  if (need > scratch_bytes)
    return fail(PAD_ERR_WORKSPACE,
                "this shape needs %zu bytes of split scratch; the static array holds %zu (use fewer splits or "
                "pad_decode)",
                need, scratch_bytes);
  void *base = nullptr;
  if ((st = scratch_address(&base)) != PAD_OK) return st;
  if (pr.cl.total > 0) {
    // the array outlives every call and keeps whatever the last one left
    cudaError_t e = cudaMemsetAsync(base, 0, pr.cl.total, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(control block)");
  }
  bind_buffers(pr, pr.ws.total > 0 ? static_cast<char *>(base) + pr.cl.total : nullptr, base);
  return run(pr, stream);
}
}  // namespace pad

extern "C" {

int32_t pad_abi_version(void) { return PAD_ABI_VERSION; }

const char *pad_status_string(pad_status st) {
  switch (st) {
    case PAD_OK: return "PAD_OK";
    case PAD_ERR_INVALID_ARG: return "PAD_ERR_INVALID_ARG";
    case PAD_ERR_UNSUPPORTED: return "PAD_ERR_UNSUPPORTED";
    case PAD_ERR_WORKSPACE: return "PAD_ERR_WORKSPACE";
    case PAD_ERR_CUDA: return "PAD_ERR_CUDA";
    case PAD_ERR_DEVICE_CHECK: return "PAD_ERR_DEVICE_CHECK";
  }
  return "PAD_ERR_UNKNOWN";
}

const char *pad_last_error(void) { return g_last_error.c_str(); }

pad_status pad_decode_plan(int64_t batch, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                           int64_t block_size, int64_t max_blocks_per_seq, int32_t num_splits, int32_t device,
                           pad_plan *plan) {
  return pad_decode_plan_ex(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_splits,
                            PAD_BF16, device, plan);
}

pad_status pad_decode_plan_ex(int64_t batch, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                              int64_t block_size, int64_t max_blocks_per_seq, int32_t num_splits, int32_t kv_dtype,
                              int32_t device, pad_plan *plan) {
  if (plan == nullptr) return fail(PAD_ERR_INVALID_ARG, "plan is NULL");
  if (kv_dtype != PAD_BF16 && kv_dtype != PAD_FP8_E4M3)
    return fail(PAD_ERR_INVALID_ARG, "kv_dtype must be PAD_BF16 or PAD_FP8_E4M3 (got %d)", kv_dtype);
  Shape s{batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
          num_kv_heads > 0 ? num_q_heads / num_kv_heads : 0, kv_dtype == PAD_FP8_E4M3};
  pad_status st = check_shape(s, num_splits);
  if (st != PAD_OK) return st;
  if (device < 0) {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) {
      cudaGetLastError();
      d = -1;
    }
    device = d;
  }
  make_plan(s, num_splits, device, plan);
  if (batch * num_kv_heads * plan->head_tiles * (int64_t)plan->num_splits > 0x7fffffffll)
    return fail(PAD_ERR_UNSUPPORTED, "too many work units for one launch");
  return PAD_OK;
}

pad_status pad_decode(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                      const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                      int32_t num_splits, pad_tensor *out, pad_tensor *lse, void *stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  Prepared pr;
  bool empty = false;
  pad_status st = prepare(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits, out, lse, &pr, &empty);
  if (st != PAD_OK || empty) return st;
  void *ws = nullptr, *ctl = nullptr;
  if (pr.ws.total > 0 && (st = get_buffer(g_ws, pr.device, stream, pr.ws.total, &ws)) != PAD_OK) return st;
  if (pr.cl.total > 0 && (st = get_buffer(g_ctl, pr.device, stream, pr.cl.total, &ctl)) != PAD_OK) return st;
  bind_buffers(pr, ws, ctl);
  return run(pr, stream);
}

pad_status pad_decode_ex(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                         const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                         int32_t num_splits, const pad_decode_options *options, pad_tensor *out, pad_tensor *lse,
                         void *stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  Prepared pr;
  bool empty = false;
  pad_status st =
      prepare(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits, out, lse, &pr, &empty, false, options);
  if (st != PAD_OK || empty) return st;
  void *ws = nullptr, *ctl = nullptr;
  if (pr.ws.total > 0 && (st = get_buffer(g_ws, pr.device, stream, pr.ws.total, &ws)) != PAD_OK) return st;
  if (pr.cl.total > 0 && (st = get_buffer(g_ctl, pr.device, stream, pr.cl.total, &ctl)) != PAD_OK) return st;
  bind_buffers(pr, ws, ctl);
  return run(pr, stream);
}

pad_status pad_decode_tcgen05(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                              const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                              int32_t num_splits, pad_tensor *out, pad_tensor *lse, void *stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  Prepared pr;
  bool empty = false;
  pad_status st = prepare(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits, out, lse, &pr, &empty, true);
  if (st != PAD_OK || empty) return st;
  void *ws = nullptr, *ctl = nullptr;
  if (pr.ws.total > 0 && (st = get_buffer(g_ws, pr.device, stream, pr.ws.total, &ws)) != PAD_OK) return st;
  if (pr.cl.total > 0 && (st = get_buffer(g_ctl, pr.device, stream, pr.cl.total, &ctl)) != PAD_OK) return st;
  bind_buffers(pr, ws, ctl);
  return run(pr, stream);
}

pad_status pad_decode_with_workspace(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                                     const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                                     int32_t num_splits, pad_tensor *out, pad_tensor *lse, void *workspace,
                                     size_t workspace_bytes, void *stream_) {
  return pad_decode_with_workspace_ex(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits, nullptr, out,
                                      lse, workspace, workspace_bytes, stream_);
}

pad_status pad_decode_with_workspace_ex(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                                        const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                                        int32_t num_splits, const pad_decode_options *options, pad_tensor *out,
                                        pad_tensor *lse, void *workspace, size_t workspace_bytes, void *stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  Prepared pr;
  bool empty = false;
  pad_status st =
      prepare(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits, out, lse, &pr, &empty, false, options);
  if (st != PAD_OK || empty) return st;
  if ((st = check_caller_buffer(pr, workspace, workspace_bytes, pr.ws.total, "workspace")) != PAD_OK) return st;
  void *ctl = nullptr;
  if (pr.cl.total > 0 && (st = get_buffer(g_ctl, pr.device, stream, pr.cl.total, &ctl)) != PAD_OK) return st;
  bind_buffers(pr, workspace, ctl);
  return run(pr, stream);
}

pad_status pad_last_launch(pad_launch_witness *w) {
  if (w == nullptr) return fail(PAD_ERR_INVALID_ARG, "witness is NULL");
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  pad::LaunchWitness *dw = nullptr;
  if ((e = pad::device_witness(device, &dw)) != cudaSuccess) return cuda_fail(e, "launch witness");
  if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  pad::LaunchWitness h{};
  if ((e = cudaMemcpy(&h, dw, sizeof(h), cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(e, "read witness");
  w->kernel = h.kernel;
  w->head_dim = h.head_dim;
  w->heads_per_tile = h.heads_per_tile;
  w->kv_dtype = h.kv_dtype;
  w->stages = h.stages;
  w->stage_tokens = h.stage_tokens;
  w->num_splits = h.num_splits;
  w->partition_tokens = h.partition_tokens;
  w->ctas = h.ctas;
  w->warps = h.warps;
  w->ctas_per_sm = h.ctas_per_sm;
  return PAD_OK;
}

pad_status pad_check_device_errors(void *stream_, uint32_t *bits) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int device = 0;
  if ((e = cudaGetDevice(&device)) != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  uint32_t *word = nullptr;
  if ((e = pad::device_error_word(device, &word)) != cudaSuccess) return cuda_fail(e, "error word");
  uint32_t v = 0;
  if ((e = cudaMemcpy(&v, word, 4, cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(e, "read error word");
  const uint32_t zero = 0;
  if ((e = cudaMemcpy(word, &zero, 4, cudaMemcpyHostToDevice)) != cudaSuccess) return cuda_fail(e, "clear error word");
  if (bits != nullptr) *bits = v;
  if (v & pad::kErrTimeout) {
    // an abandoned launch may have left merge counters set: re-zero the
    // library's own control blocks on this device
    std::lock_guard<std::mutex> lock(g_ws_mu);
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    for (auto &kv : g_ctl)
      if (kv.first.first == device && kv.second.ptr != nullptr) cudaMemset(kv.second.ptr, 0, kv.second.bytes);
  }
  if (v != 0)
    return fail(PAD_ERR_DEVICE_CHECK, "kernel saw %s%s%s", (v & pad::kErrBlockId) ? "an out-of-range block id; " : "",
                (v & pad::kErrSeqLen) ? "an out-of-range sequence length; " : "",
                (v & pad::kErrTimeout) ? "a bounded wait that gave up (a stage whose copies never completed: an "
                                         "internal error; or the failure-path test hook)" : "");
  return PAD_OK;
}

pad_status pad_inject_stage_timeout(int32_t partition) {
  if (partition < -1 || partition >= pad::kMaxSplits)
    return fail(PAD_ERR_INVALID_ARG, "partition must be -1 (none) or in [0, %d) (got %d)", pad::kMaxSplits, partition);
  g_stall_partition = partition;
  return PAD_OK;
}

pad_status pad_release_workspace(int32_t device) {
  std::lock_guard<std::mutex> lock(g_ws_mu);
  int cur = 0;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  for (auto *pool : {&g_ws, &g_ctl}) {
    for (auto it = pool->begin(); it != pool->end();) {
      if (device >= 0 && it->first.first != device) {
        ++it;
        continue;
      }
      if ((e = cudaSetDevice(it->first.first)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
      if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
      if (it->second.ptr != nullptr) cudaFree(it->second.ptr);
      it = pool->erase(it);
    }
  }
  if ((e = cudaSetDevice(cur)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  return PAD_OK;
}

}  // extern "C"
