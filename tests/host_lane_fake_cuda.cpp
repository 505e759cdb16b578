// Host logic of the C ABI against a fake CUDA runtime (CPU, no GPU).
//
// tests/test_host_sanitizers.py compiles the library's host file (pad_api.cpp,
// unchanged) with this file under -fsanitize=address,undefined.  This file
// supplies, in place of the CUDA runtime and of the library's kernel module,
// fakes of exactly the calls pad_api.cpp makes: "device" memory is host memory
// registered here, streams are plain handles, the tensor-map encoder checks the
// documented cuTensorMapEncodeTiled constraints and records each map, and a
// "launch" records the parameter block instead of running a kernel.  Failures
// are injected by the fakes (an allocation that fails, a launch that fails, an
// encoder that refuses, no device, a stream under capture, error bits set by a
// "kernel"), never by a GPU.  The driver below checks what the library hands
// to the kernel -- pointers, strides, plan, scratch placement, tensor maps --
// and how every failure comes back: status, message, nothing launched.
//
// Run without arguments for every scenario; with "no-encoder" for the one
// that needs a process whose driver lacks the encoder (the library looks it up
// once per process).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "pad.h"
#include "pad_internal.h"

// ---------------------------------------------------------------- the fakes --

namespace fake {
struct Alloc {
  char *base;
  size_t bytes;
  int device;
  bool library;  // allocated through cudaMalloc (the library's own)
};
std::vector<Alloc> allocs;
int current_device = 0;
bool no_device = false;
int malloc_failures = 0;  // the next N cudaMalloc calls fail
bool capturing = false;
bool no_encoder = false;
bool encoder_refuses = false;
cudaError_t launch_result = cudaSuccess;
std::vector<std::string> events;  // "malloc N", "free", "sync", "devsync", "memset N"
struct Launch {
  pad::PartitionParams p;
  int D, hpt, grid, ctas_per_sm;
  bool fp8, umma;
  cudaStream_t stream;
};
std::vector<Launch> launches;
// schedule passes: the parameter block each was given and its stream
std::vector<std::pair<pad::PartitionParams, cudaStream_t>> schedules;
struct Encode {
  CUtensorMapDataType dt;
  cuuint32_t rank;
  void *addr;
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5];
  CUtensorMapSwizzle swizzle;
};
std::vector<Encode> encodes;
std::vector<std::string> encoder_violations;
uint32_t err_word = 0;
pad::LaunchWitness witness{};

void *device_buffer(size_t bytes, int device = 0) {  // an input: registered, not counted
  char *p = static_cast<char *>(aligned_alloc(256, (bytes + 255) / 256 * 256));
  memset(p, 0, bytes);
  allocs.push_back({p, bytes, device, false});
  return p;
}
const Alloc *find(const void *p) {
  for (const Alloc &a : allocs)
    if (static_cast<const char *>(p) >= a.base && static_cast<const char *>(p) < a.base + (a.bytes ? a.bytes : 1))
      return &a;
  return nullptr;
}
int library_live() {
  int n = 0;
  for (const Alloc &a : allocs) n += a.library;
  return n;
}
}  // namespace fake

cudaError_t cudaGetDevice(int *d) {
  if (fake::no_device) return cudaErrorNoDevice;
  *d = fake::current_device;
  return cudaSuccess;
}
cudaError_t cudaSetDevice(int d) {
  fake::current_device = d;
  return cudaSuccess;
}
cudaError_t cudaDeviceGetAttribute(int *v, enum cudaDeviceAttr a, int) {
  if (a != cudaDevAttrMultiProcessorCount) return cudaErrorInvalidValue;
  *v = 148;
  return cudaSuccess;
}
cudaError_t cudaGetLastError(void) { return cudaSuccess; }
const char *cudaGetErrorString(cudaError_t e) {
  static thread_local char buf[64];
  snprintf(buf, sizeof buf, "fake CUDA error %d", (int)e);
  return buf;
}
cudaError_t cudaPointerGetAttributes(struct cudaPointerAttributes *a, const void *p) {
  memset(a, 0, sizeof(*a));
  const fake::Alloc *al = fake::find(p);
  a->type = al ? cudaMemoryTypeDevice : cudaMemoryTypeUnregistered;
  a->device = al ? al->device : -2;
  return cudaSuccess;
}
cudaError_t cudaStreamIsCapturing(cudaStream_t, enum cudaStreamCaptureStatus *st) {
  *st = fake::capturing ? cudaStreamCaptureStatusActive : cudaStreamCaptureStatusNone;
  return cudaSuccess;
}
cudaError_t cudaStreamSynchronize(cudaStream_t) {
  fake::events.push_back("sync");
  return cudaSuccess;
}
cudaError_t cudaDeviceSynchronize(void) {
  fake::events.push_back("devsync");
  return cudaSuccess;
}
cudaError_t cudaMalloc(void **p, size_t n) {
  if (fake::malloc_failures > 0) {
    --fake::malloc_failures;
    fake::events.push_back("malloc-failed " + std::to_string(n));
    return cudaErrorMemoryAllocation;
  }
  char *q = static_cast<char *>(aligned_alloc(256, (n + 255) / 256 * 256));
  memset(q, 0xCD, n);  // not zero: the library must clear what needs clearing
  fake::allocs.push_back({q, n, fake::current_device, true});
  fake::events.push_back("malloc " + std::to_string(n));
  *p = q;
  return cudaSuccess;
}
cudaError_t cudaFree(void *p) {
  for (size_t i = 0; i < fake::allocs.size(); ++i)
    if (fake::allocs[i].base == p) {
      free(p);
      fake::allocs.erase(fake::allocs.begin() + (long)i);
      fake::events.push_back("free");
      return cudaSuccess;
    }
  fake::events.push_back("free-unknown");
  return cudaErrorInvalidValue;
}
static cudaError_t fake_memset(void *p, int v, size_t n) {
  const fake::Alloc *a = fake::find(p);
  if (a == nullptr || static_cast<char *>(p) + n > a->base + a->bytes) {
    fake::events.push_back("memset-out-of-range");
    return cudaErrorInvalidValue;
  }
  memset(p, v, n);
  fake::events.push_back("memset " + std::to_string(n));
  return cudaSuccess;
}
cudaError_t cudaMemsetAsync(void *p, int v, size_t n, cudaStream_t) { return fake_memset(p, v, n); }
cudaError_t cudaMemset(void *p, int v, size_t n) { return fake_memset(p, v, n); }
cudaError_t cudaMemcpy(void *d, const void *s, size_t n, enum cudaMemcpyKind) {
  memcpy(d, s, n);
  return cudaSuccess;
}

// cuTensorMapEncodeTiled's documented argument rules (CUDA driver API), checked
// on every map the library asks for.
static CUresult fake_encode(CUtensorMap *map, CUtensorMapDataType dt, cuuint32_t rank, void *addr,
                            const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box,
                            const cuuint32_t *elem, CUtensorMapInterleave il, CUtensorMapSwizzle sw,
                            CUtensorMapL2promotion, CUtensorMapFloatOOBfill) {
  auto bad = [](const std::string &why) {
    fake::encoder_violations.push_back(why);
    return CUDA_ERROR_INVALID_VALUE;
  };
  if (fake::encoder_refuses) return CUDA_ERROR_INVALID_VALUE;
  const cuuint64_t esize = dt == CU_TENSOR_MAP_DATA_TYPE_UINT8 ? 1 : 2;
  if (rank < 1 || rank > 5) return bad("rank");
  if (reinterpret_cast<uintptr_t>(addr) % 16) return bad("global address not 16-byte aligned");
  if (fake::find(addr) == nullptr) return bad("global address is not device memory");
  for (cuuint32_t i = 0; i < rank; ++i) {
    if (dims[i] == 0 || dims[i] > (1ull << 32)) return bad("dim out of range");
    if (box[i] == 0 || box[i] > 256) return bad("box dim out of [1, 256]");
    if (box[i] > dims[i]) return bad("box larger than the tensor");
    if (elem[i] < 1 || elem[i] > 8) return bad("element stride");
  }
  for (cuuint32_t i = 0; i + 1 < rank; ++i)
    if (strides[i] % 16 || strides[i] >= (1ull << 40)) return bad("global stride not a multiple of 16 below 2^40");
  if ((box[0] * esize) % 16) return bad("inner box bytes not a multiple of 16");
  if (il != CU_TENSOR_MAP_INTERLEAVE_NONE) return bad("interleave");
  const cuuint64_t span = sw == CU_TENSOR_MAP_SWIZZLE_128B ? 128 : sw == CU_TENSOR_MAP_SWIZZLE_64B ? 64
                          : sw == CU_TENSOR_MAP_SWIZZLE_32B ? 32 : 0;
  if (span && box[0] * esize > span) return bad("inner box wider than the swizzle span");
  fake::Encode e{};
  e.dt = dt;
  e.rank = rank;
  e.addr = addr;
  for (cuuint32_t i = 0; i < rank; ++i) e.dims[i] = dims[i], e.box[i] = box[i];
  for (cuuint32_t i = 0; i + 1 < rank; ++i) e.strides[i] = strides[i];
  e.swizzle = sw;
  fake::encodes.push_back(e);
  memset(map, 0xAB, sizeof(*map));
  return CUDA_SUCCESS;
}
cudaError_t cudaGetDriverEntryPoint(const char *sym, void **fn, unsigned long long,
                                    enum cudaDriverEntryPointQueryResult *q) {
  if (fake::no_encoder || strcmp(sym, "cuTensorMapEncodeTiled") != 0) {
    *fn = nullptr;
    if (q) *q = cudaDriverEntryPointSymbolNotFound;
    return cudaSuccess;
  }
  *fn = reinterpret_cast<void *>(&fake_encode);
  if (q) *q = cudaDriverEntryPointSuccess;
  return cudaSuccess;
}

// The kernel module's entry points: a launch is recorded, and the witness
// record is written as the kernels write theirs.
namespace pad {
int partition_stages(int D, int hpt, bool f8) { return stages_for(D, hpt, f8); }
int umma_stages() { return 1; }
cudaError_t device_error_word(int, uint32_t **ptr) {
  *ptr = &fake::err_word;
  return cudaSuccess;
}
cudaError_t device_witness(int, LaunchWitness **ptr) {
  *ptr = &fake::witness;
  return cudaSuccess;
}
cudaError_t launch_partition(const PartitionParams &p, int D, int hpt, bool f8, int grid, int cps, cudaStream_t s) {
  if (fake::launch_result != cudaSuccess) return fake::launch_result;
  // the instances the kernel module has: the fixed residency, and the dense
  // build of the E4M3 8-head tile at D = 128
  if (cps != ctas_per_sm_for(D, hpt, f8) && !(has_dense_build(D, hpt, f8) && cps == kDenseCtasPerSm))
    return cudaErrorInvalidValue;
  fake::launches.push_back({p, D, hpt, grid, cps, f8, false, s});
  fake::witness = LaunchWitness{1, D, hpt, f8 ? (int32_t)PAD_FP8_E4M3 : (int32_t)PAD_BF16, stages_for(D, hpt, f8),
                                stage_tokens_for(D, hpt, f8), p.S, p.P, grid, warps_for(D, hpt, f8), cps};
  return cudaSuccess;
}
cudaError_t launch_schedule(const PartitionParams &p, cudaStream_t s) {
  if (fake::launch_result != cudaSuccess) return fake::launch_result;
  fake::schedules.push_back({p, s});
  return cudaSuccess;
}
cudaError_t launch_umma(const PartitionParams &p, int grid, cudaStream_t s) {
  if (fake::launch_result != cudaSuccess) return fake::launch_result;
  fake::launches.push_back({p, 128, 32, grid, kUmmaCtasPerSm, false, true, s});
  fake::witness = LaunchWitness{2, 128, 32, (int32_t)PAD_BF16, 1, kUmmaStageTokens, p.S, p.P, grid, kUmmaWarps,
                                kUmmaCtasPerSm};
  return cudaSuccess;
}
}  // namespace pad

// ------------------------------------------------------------------ driver --

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

static bool message_has(const char *needle) { return strstr(pad_last_error(), needle) != nullptr; }

static pad_tensor tensor(void *data, int32_t dtype, std::vector<int64_t> shape) {
  pad_tensor t;
  memset(&t, 0, sizeof(t));
  t.data = data;
  t.dtype = dtype;
  t.ndim = (int32_t)shape.size();
  int64_t s = 1;
  for (int i = t.ndim - 1; i >= 0; --i) {
    t.shape[i] = shape[i];
    t.stride[i] = s;
    s *= shape[i];
  }
  return t;
}

// One decode problem with every buffer in fake device memory.
struct Problem {
  int64_t B, Hq, Hkv, D, bs, W, NB;
  bool fp8, nhd;
  pad_tensor q, k, v, tables, lens, out, lse;
  Problem(int64_t B_, int64_t Hq_, int64_t Hkv_, int64_t D_, int64_t bs_, int64_t W_, bool fp8_ = false,
          bool nhd_ = false)
      : B(B_), Hq(Hq_), Hkv(Hkv_), D(D_), bs(bs_), W(W_), NB(B_ * W_ + 1), fp8(fp8_), nhd(nhd_) {
    const int64_t eb = fp8 ? 1 : 2, kv = NB * Hkv * bs * D;
    q = tensor(fake::device_buffer(B * Hq * D * 2), PAD_BF16, {B, Hq, D});
    const int32_t kvt = fp8 ? PAD_FP8_E4M3 : PAD_BF16;
    k = tensor(fake::device_buffer(kv * eb), kvt, {NB, Hkv, bs, D});
    v = tensor(fake::device_buffer(kv * eb), kvt, {NB, Hkv, bs, D});
    if (nhd) {  // storage [NB, bs, Hkv, D], seen as [NB, Hkv, bs, D]
      for (pad_tensor *t : {&k, &v}) {
        t->stride[1] = D;
        t->stride[2] = Hkv * D;
      }
    }
    tables = tensor(fake::device_buffer(B * W * 4), PAD_I32, {B, W});
    lens = tensor(fake::device_buffer(B * 4), PAD_I32, {B});
    out = tensor(fake::device_buffer(B * Hq * D * 2), PAD_BF16, {B, Hq, D});
    lse = tensor(fake::device_buffer(B * Hq * 4), PAD_F32, {B, Hq});
  }
  pad_status decode(int32_t splits, void *stream, const pad_decode_options *o = nullptr) {
    return o ? pad_decode_ex(&q, &k, &v, &tables, &lens, 0.125f, splits, o, &out, &lse, stream)
             : pad_decode(&q, &k, &v, &tables, &lens, 0.125f, splits, &out, &lse, stream);
  }
  pad_plan plan(int32_t splits) const {
    pad_plan p;
    memset(&p, 0, sizeof(p));
    pad_decode_plan_ex(B, Hq, Hkv, D, bs, W, splits, fp8 ? PAD_FP8_E4M3 : PAD_BF16, 0, &p);
    return p;
  }
};

static bool inside(const void *p, size_t bytes, const fake::Alloc *a) {
  return a != nullptr && static_cast<const char *>(p) >= a->base &&
         static_cast<const char *>(p) + bytes <= a->base + a->bytes;
}

// What the library handed to the kernel for `pr` with `splits`.
static void check_launch(const Problem &pr, int32_t splits, const fake::Launch &L, cudaStream_t s, const char *what) {
  const pad_plan pl = pr.plan(splits);
  const pad::PartitionParams &p = L.p;
  CHECK(L.grid == pl.ctas && (uint32_t)pl.ctas == p.n_units, "%s: grid %d, plan %d", what, L.grid, pl.ctas);
  CHECK(L.stream == s, "%s: launched on another stream", what);
  CHECK(L.D == pr.D && L.hpt == pl.heads_per_tile && L.fp8 == pr.fp8 && L.ctas_per_sm == pl.ctas_per_sm,
        "%s: kernel instance", what);
  CHECK(p.S == pl.num_splits && p.P == pl.partition_tokens && p.HT == pl.head_tiles, "%s: plan fields", what);
  CHECK(p.B == pr.B && p.Hq == pr.Hq && p.Hkv == pr.Hkv && p.g == pr.Hq / pr.Hkv, "%s: sizes", what);
  CHECK((1 << p.bs_log2) == pr.bs && p.max_blocks == pr.W && p.num_blocks == pr.NB, "%s: table sizes", what);
  CHECK(p.q == pr.q.data && p.k == pr.k.data && p.v == pr.v.data && p.tables == pr.tables.data &&
            p.seq_lens == pr.lens.data && p.out == pr.out.data && p.lse == pr.lse.data,
        "%s: tensor pointers", what);
  CHECK(p.k_sblk == pr.k.stride[0] && p.k_sh == pr.k.stride[1] && p.k_ss == pr.k.stride[2] &&
            p.v_ss == pr.v.stride[2] && p.q_sb == pr.q.stride[0] && p.o_sh == pr.out.stride[1],
        "%s: strides", what);
  CHECK(p.err == &fake::err_word && p.witness == &fake::witness, "%s: error word / witness", what);
  if (p.S > 1) {
    const size_t ob = (size_t)(pr.B * pr.Hq * p.S * pr.D * 4), lb = (size_t)(pr.B * pr.Hq * p.S * 4);
    const fake::Alloc *a = fake::find(p.o_part);
    CHECK(inside(p.o_part, ob, a) && inside(p.lse_part, lb, a), "%s: partials outside their buffer", what);
    CHECK((const char *)p.lse_part >= (const char *)p.o_part + ob, "%s: partial regions overlap", what);
    // the unit order: after the partials, in the same buffer, written by a
    // schedule pass launched just before on the same stream with the same order
    const bool sched = pad::schedules_units(pr.B, p.S, p.P, pl.heads_per_tile);
    CHECK((p.order != nullptr) == sched, "%s: unit order %s", what, sched ? "missing" : "unexpected");
    if (sched) {
      CHECK(inside(p.order, (size_t)p.n_units * 4, a) && (const char *)p.order >= (const char *)p.lse_part + lb,
            "%s: unit order outside its place", what);
      CHECK(!fake::schedules.empty() && fake::schedules.back().first.order == p.order &&
                fake::schedules.back().second == L.stream && fake::schedules.back().first.n_units == p.n_units,
            "%s: no schedule pass before the launch", what);
    }
    const size_t cb = (size_t)(pr.B * pr.Hkv * p.HT * 4);
    const fake::Alloc *c = fake::find(p.counters);
    CHECK(inside(p.counters, cb, c) && c != a, "%s: counters outside their own buffer", what);
    bool zero = true;
    for (size_t i = 0; c && i < cb / 4; ++i) zero = zero && p.counters[i] == 0;
    CHECK(zero, "%s: merge counters not zero at launch", what);
  } else {
    CHECK(p.o_part == nullptr && p.lse_part == nullptr && p.counters == nullptr && p.order == nullptr,
          "%s: scratch with S == 1", what);
  }
}

// The two cache maps of the last launch: the 5-D view of the caller's strides.
static void check_cache_maps(const Problem &pr, size_t first, const char *what) {
  CHECK(fake::encodes.size() >= first + 2, "%s: %zu maps", what, fake::encodes.size() - first);
  const int64_t eb = pr.fp8 ? 1 : 2, rowb = pr.D * eb, rw = rowb < 128 ? rowb : 128;
  const pad_plan pl = pr.plan(0);
  for (int i = 0; i < 2 && fake::encodes.size() >= first + 2; ++i) {
    const fake::Encode &e = fake::encodes[first + i];
    const pad_tensor &t = i == 0 ? pr.k : pr.v;
    CHECK(e.addr == t.data && e.rank == 5, "%s: map %d address/rank", what, i);
    CHECK(e.dt == (pr.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16), "%s: map dtype", what);
    CHECK(e.dims[0] * eb == (cuuint64_t)rw && e.dims[1] == (cuuint64_t)pr.bs && e.dims[2] * rw == (cuuint64_t)rowb &&
              e.dims[3] == (cuuint64_t)pr.Hkv && e.dims[4] == (cuuint64_t)pr.NB,
          "%s: map %d dims", what, i);
    CHECK(e.strides[0] == (cuuint64_t)(t.stride[2] * eb) && e.strides[1] == (cuuint64_t)rw &&
              e.strides[2] == (cuuint64_t)(t.stride[1] * eb) && e.strides[3] == (cuuint64_t)(t.stride[0] * eb),
          "%s: map %d strides", what, i);
    const int64_t rows = pr.bs < pl.stage_tokens ? pr.bs : pl.stage_tokens;
    CHECK(e.box[0] == e.dims[0] && e.box[1] == (cuuint32_t)rows && e.box[2] == e.dims[2] && e.box[3] == 1 &&
              e.box[4] == 1,
          "%s: map %d box", what, i);
    CHECK(e.swizzle == (rw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B), "%s: swizzle", what);
  }
}

static void scenarios() {
  cudaStream_t s1 = reinterpret_cast<cudaStream_t>(0x1001), s2 = reinterpret_cast<cudaStream_t>(0x2002);

  // a split decode: scratch allocated and cleared, parameters bound, maps encoded
  Problem a(3, 8, 2, 128, 16, 8);
  size_t enc0 = fake::encodes.size();
  CHECK(a.decode(4, s1) == PAD_OK, "split decode: %s", pad_last_error());
  CHECK(fake::launches.size() == 1, "one launch");
  if (!fake::launches.empty()) check_launch(a, 4, fake::launches.back(), s1, "split decode");
  check_cache_maps(a, enc0, "split decode");
  CHECK(fake::library_live() == 2, "partials and control buffers: %d live", fake::library_live());
  pad_launch_witness w;
  CHECK(pad_last_launch(&w) == PAD_OK && w.kernel == 1 && w.num_splits == a.plan(4).num_splits &&
            w.ctas == a.plan(4).ctas && w.ctas_per_sm == a.plan(4).ctas_per_sm && w.ctas_per_sm == 5,
        "witness read back");


  // the same shape again: no new allocation
  size_t ev = fake::events.size();
  CHECK(a.decode(4, s1) == PAD_OK && fake::launches.size() == 2, "repeat decode");
  for (size_t i = ev; i < fake::events.size(); ++i)
    CHECK(fake::events[i].rfind("malloc", 0) != 0, "repeat decode allocated (%s)", fake::events[i].c_str());

  // heavy units (2048-token partitions of a 32-head tile): a schedule pass on
  // the same stream writes the unit order into the partials buffer first
  Problem heavy(2, 32, 1, 128, 16, 256);
  const size_t sched0 = fake::schedules.size();
  CHECK(heavy.decode(2, s1) == PAD_OK && fake::schedules.size() == sched0 + 1, "scheduled decode: %s",
        pad_last_error());
  CHECK(heavy.plan(2).partition_tokens * heavy.plan(2).heads_per_tile >= 32768, "heavy units");
  if (!fake::launches.empty()) check_launch(heavy, 2, fake::launches.back(), s1, "scheduled decode");
  CHECK(a.decode(4, s1) == PAD_OK && fake::schedules.size() == sched0 + 1, "light units scheduled");

  // one partition: no scratch at all
  Problem one(2, 8, 2, 128, 16, 4);
  CHECK(one.decode(1, s1) == PAD_OK, "S == 1 decode");
  if (!fake::launches.empty()) check_launch(one, 1, fake::launches.back(), s1, "S == 1 decode");

  // a larger shape on the same stream: the stream is drained before the old buffer is freed
  Problem big(12, 8, 2, 128, 16, 32);
  ev = fake::events.size();
  CHECK(big.decode(16, s1) == PAD_OK, "growing decode: %s", pad_last_error());
  int sync_at = -1, free_at = -1;
  for (size_t i = ev; i < fake::events.size(); ++i) {
    if (fake::events[i] == "sync" && sync_at < 0) sync_at = (int)i;
    if (fake::events[i] == "free" && free_at < 0) free_at = (int)i;
  }
  CHECK(free_at >= 0 && sync_at >= 0 && sync_at < free_at, "old scratch freed before the stream drained");
  if (!fake::launches.empty()) check_launch(big, 16, fake::launches.back(), s1, "growing decode");

  // under capture: a call that fits runs; one that needs more scratch is refused, nothing launched
  fake::capturing = true;
  size_t nl = fake::launches.size();
  CHECK(a.decode(4, s1) == PAD_OK && fake::launches.size() == nl + 1, "capture-safe call");
  Problem bigger(40, 8, 2, 128, 16, 64);
  nl = fake::launches.size();
  CHECK(bigger.decode(32, s1) == PAD_ERR_WORKSPACE && message_has("captured"), "growth under capture: %s",
        pad_last_error());
  CHECK(fake::launches.size() == nl, "launched under a refused capture");
  fake::capturing = false;

  // another stream: its own scratch
  const int live = fake::library_live();
  CHECK(a.decode(4, s2) == PAD_OK && fake::library_live() == live + 2, "second stream scratch");
  if (fake::launches.size() >= 2) {
    const pad::PartitionParams &p2 = fake::launches.back().p;
    const pad::PartitionParams &p1 = fake::launches[fake::launches.size() - 2].p;
    CHECK(fake::find(p2.o_part) != fake::find(p1.o_part), "two streams share partials");
  }

  // NHD cache and E4M3 caches: the maps follow the caller's strides and element size
  Problem nhd(2, 16, 4, 128, 16, 6, false, true);
  enc0 = fake::encodes.size();
  CHECK(nhd.decode(0, s1) == PAD_OK, "NHD decode: %s", pad_last_error());
  check_cache_maps(nhd, enc0, "NHD decode");
  pad_decode_options o;
  memset(&o, 0, sizeof(o));
  o.k_scale = 0.046875f;
  o.v_scale = 0.01953125f;
  for (int64_t D : {64, 128, 256}) {
    Problem f8(2, 8, 2, D, 16, 6, true);
    enc0 = fake::encodes.size();
    CHECK(f8.decode(3, s1, &o) == PAD_OK, "E4M3 D=%lld decode: %s", (long long)D, pad_last_error());
    check_cache_maps(f8, enc0, "E4M3 decode");
    if (!fake::launches.empty()) {
      const pad::PartitionParams &p = fake::launches.back().p;
      CHECK(p.v_scale == o.v_scale && std::fabs(p.scale_log2 - (float)(0.125 * 0.046875 * 1.4426950408889634)) == 0.f,
            "E4M3 scales folded");
    }
  }

  // window and sinks reach the kernel; sinks must be device memory
  float *sinks = static_cast<float *>(fake::device_buffer(8 * 4));
  pad_tensor st = tensor(sinks, PAD_F32, {8});
  memset(&o, 0, sizeof(o));
  o.window_left = 100;
  o.sinks = &st;
  CHECK(a.decode(0, s1, &o) == PAD_OK && fake::launches.back().p.window == 100 && fake::launches.back().p.sinks == sinks,
        "window and sinks bound");
  float host_sinks[8] = {0};
  pad_tensor hst = tensor(host_sinks, PAD_F32, {8});
  o.sinks = &hst;
  CHECK(a.decode(0, s1, &o) == PAD_ERR_INVALID_ARG && message_has("sinks"), "host sinks accepted");

  // device-pointer checks: host memory, another device's memory
  Problem h(2, 8, 2, 128, 16, 4);
  uint16_t host_q[2 * 8 * 128];
  h.q.data = host_q;
  CHECK(h.decode(0, s1) == PAD_ERR_INVALID_ARG && message_has("q: must be device memory"), "host q: %s",
        pad_last_error());
  h.q.data = fake::device_buffer(2 * 8 * 128 * 2, 1);
  CHECK(h.decode(0, s1) == PAD_ERR_INVALID_ARG && message_has("lives on device 1"), "q on device 1: %s",
        pad_last_error());

  // caller-owned partials
  const pad_plan pa = a.plan(4);
  void *ws = fake::device_buffer((size_t)pa.workspace_bytes + 512);
  nl = fake::launches.size();
  CHECK(pad_decode_with_workspace(&a.q, &a.k, &a.v, &a.tables, &a.lens, 0.125f, 4, &a.out, &a.lse, ws,
                                  (size_t)pa.workspace_bytes - 1, s1) == PAD_ERR_INVALID_ARG,
        "short workspace accepted");
  CHECK(pad_decode_with_workspace(&a.q, &a.k, &a.v, &a.tables, &a.lens, 0.125f, 4, &a.out, &a.lse,
                                  static_cast<char *>(ws) + 16, (size_t)pa.workspace_bytes, s1) == PAD_ERR_INVALID_ARG,
        "misaligned workspace accepted");
  char host_ws[4096];
  CHECK(pad_decode_with_workspace(&a.q, &a.k, &a.v, &a.tables, &a.lens, 0.125f, 4, &a.out, &a.lse, host_ws,
                                  sizeof(host_ws), s1) != PAD_OK,
        "host workspace accepted");
  CHECK(fake::launches.size() == nl, "a refused workspace call launched");
  CHECK(pad_decode_with_workspace(&a.q, &a.k, &a.v, &a.tables, &a.lens, 0.125f, 4, &a.out, &a.lse, ws,
                                  (size_t)pa.workspace_bytes, s1) == PAD_OK &&
            fake::find(fake::launches.back().p.o_part) == fake::find(ws),
        "caller workspace not used");

  // the tcgen05 entry: its own maps (8-row boxes, q map), and its envelope
  Problem tc(2, 32, 1, 128, 16, 8);
  enc0 = fake::encodes.size();
  CHECK(pad_decode_tcgen05(&tc.q, &tc.k, &tc.v, &tc.tables, &tc.lens, 0.125f, 2, &tc.out, &tc.lse, s1) == PAD_OK &&
            fake::launches.back().umma,
        "tcgen05 decode: %s", pad_last_error());
  CHECK(fake::encodes.size() == enc0 + 3 && fake::encodes[enc0].box[1] == 8 && fake::encodes[enc0 + 2].rank == 4 &&
            fake::encodes[enc0 + 2].box[1] == 32 && fake::encodes[enc0 + 2].addr == tc.q.data,
        "tcgen05 maps");
  CHECK(pad_last_launch(&w) == PAD_OK && w.kernel == 2, "tcgen05 witness");
  CHECK(pad_decode_tcgen05(&a.q, &a.k, &a.v, &a.tables, &a.lens, 0.125f, 2, &a.out, &a.lse, s1) ==
            PAD_ERR_UNSUPPORTED,
        "tcgen05 took a group of 4");

  // injected failures: allocation, launch, encoder, no device
  cudaStream_t s3 = reinterpret_cast<cudaStream_t>(0x3003);
  fake::malloc_failures = 2;  // the headroom request and the exact one
  nl = fake::launches.size();
  CHECK(a.decode(4, s3) == PAD_ERR_WORKSPACE && message_has("cudaMalloc"), "failed allocation: %s", pad_last_error());
  CHECK(fake::launches.size() == nl, "launched without scratch");
  fake::malloc_failures = 1;  // only the headroom request fails: the exact size is taken
  CHECK(a.decode(4, s3) == PAD_OK, "exact-size fallback: %s", pad_last_error());
  fake::launch_result = cudaErrorLaunchOutOfResources;
  CHECK(a.decode(4, s1) == PAD_ERR_CUDA && message_has("launch"), "failed launch: %s", pad_last_error());
  fake::launch_result = cudaSuccess;
  fake::encoder_refuses = true;
  nl = fake::launches.size();
  CHECK(a.decode(4, s1) == PAD_ERR_INVALID_ARG && message_has("TMA"), "refused map: %s", pad_last_error());
  CHECK(fake::launches.size() == nl, "launched without maps");
  fake::encoder_refuses = false;
  fake::no_device = true;
  CHECK(a.decode(4, s1) == PAD_ERR_CUDA && message_has("cudaGetDevice"), "no device: %s", pad_last_error());
  pad_plan pp;
  CHECK(pad_decode_plan(3, 8, 2, 128, 16, 8, 0, -1, &pp) == PAD_OK, "plan without a device");
  CHECK(pad_last_launch(&w) == PAD_ERR_CUDA, "witness without a device");
  fake::no_device = false;

  // error bits raised by a "kernel": reported once, cleared; a timeout re-zeroes the control blocks
  fake::err_word = pad::kErrBlockId | pad::kErrSeqLen;
  uint32_t bits = 0;
  CHECK(pad_check_device_errors(s1, &bits) == PAD_ERR_DEVICE_CHECK && bits == 3 && fake::err_word == 0 &&
            message_has("block id") && message_has("sequence length"),
        "error bits: %s", pad_last_error());
  CHECK(pad_check_device_errors(s1, &bits) == PAD_OK && bits == 0, "error bits not cleared");
  if (!fake::launches.empty()) {
    uint32_t *counters = fake::launches.back().p.counters;
    if (counters) counters[0] = 7;  // a launch that gave up left a count behind
    fake::err_word = pad::kErrTimeout;
    CHECK(pad_check_device_errors(s1, &bits) == PAD_ERR_DEVICE_CHECK && bits == pad::kErrTimeout,
          "timeout bit: %s", pad_last_error());
    CHECK(counters == nullptr || counters[0] == 0, "control block not re-zeroed after a timeout");
  }

  // releasing the library's buffers frees exactly them
  CHECK(pad_release_workspace(-1) == PAD_OK && fake::library_live() == 0, "release left %d buffers",
        fake::library_live());
  CHECK(a.decode(4, s1) == PAD_OK && fake::library_live() == 2, "decode after release");

  // the 8-head tiles at D = 128: the six-per-SM build from four full waves
  // at five per SM (4 * 5 * 148 = 2960 units) on, the five-per-SM one below
  pad_launch_witness w2;
  Problem e_few(23, 8, 8, 128, 16, 16, true), e_many(24, 8, 8, 128, 16, 16, true);  // 2944 / 3072 units at S = 16
  CHECK(e_few.plan(16).ctas == 2944 && e_few.plan(16).ctas_per_sm == 5, "E4M3 8-head, 2944 units: %d per SM",
        e_few.plan(16).ctas_per_sm);
  CHECK(e_many.plan(16).ctas == 3072 && e_many.plan(16).ctas_per_sm == 6, "E4M3 8-head, 3072 units: %d per SM",
        e_many.plan(16).ctas_per_sm);
  CHECK(Problem(23, 8, 8, 128, 16, 16).plan(16).ctas_per_sm == 5 && Problem(24, 8, 8, 128, 16, 16).plan(16).ctas_per_sm == 6,
        "bf16 8-head: the same two builds");
  CHECK(e_many.decode(16, s1) == PAD_OK, "dense E4M3 decode: %s", pad_last_error());
  if (!fake::launches.empty()) check_launch(e_many, 16, fake::launches.back(), s1, "dense E4M3 decode");
  CHECK(pad_last_launch(&w2) == PAD_OK && w2.ctas_per_sm == 6, "dense build witnessed");
  CHECK(e_few.decode(16, s1) == PAD_OK, "E4M3 decode: %s", pad_last_error());
  if (!fake::launches.empty()) check_launch(e_few, 16, fake::launches.back(), s1, "E4M3 decode");
  CHECK(fake::encoder_violations.empty(), "encoder rule broken: %s",
        fake::encoder_violations.empty() ? "" : fake::encoder_violations[0].c_str());
}

static void no_encoder_scenario() {
  // the library looks the encoder up once per process: this runs in its own
  fake::no_encoder = true;
  Problem a(3, 8, 2, 128, 16, 8);
  CHECK(a.decode(4, reinterpret_cast<cudaStream_t>(0x1001)) == PAD_ERR_CUDA && message_has("cuTensorMapEncodeTiled"),
        "missing encoder: %s", pad_last_error());
  CHECK(fake::launches.empty(), "launched without an encoder");
}

int main(int argc, char **argv) {
  if (argc > 1 && strcmp(argv[1], "no-encoder") == 0)
    no_encoder_scenario();
  else
    scenarios();
  for (const fake::Alloc &a : fake::allocs) free(a.base);
  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("host lane (C ABI over a fake runtime): clean\n");
  return 0;
}
