// pad_decode_static_scratch: the split-KV decode with its partition scratch in a
// fixed array compiled into the library, for callers that cannot allocate device
// memory.
//
// Who needs it: code that must not call cudaMalloc or any allocating routine at
// the point where it decodes -- for example a runtime whose memory is entirely
// pre-planned (a fixed arena carved up at start-up), a host thread that is not
// allowed to take the allocator's locks or trigger the synchronisation cudaMalloc
// and cudaFree may imply, or an embedding that has no allocator of its own to
// hand the library.  pad_decode grows library-owned scratch on demand and
// pad_decode_with_workspace needs the caller to supply scratch; this entry point
// needs neither.
//
// The scratch is one file-scope __device__ array of kStaticScratchBytes.  Every
// GPU that loads the library holds it until the process exits, and every call on
// that GPU shares it.  Host code cannot use the array's name as a device address
// (on the host it names a stand-in object), so the device address is looked up
// with cudaGetSymbolAddress, once per device, with that device current, and then
// passed to the kernels.
#include <cuda_runtime.h>
#include <stdio.h>

#include <atomic>

#include "pad.h"
#include "pad_internal.h"

// 32 MiB: enough for the split partials of e.g. B=64 sequences x 40 query heads x
// 16 partitions at head_dim 128 (64*40*16*(128+1)*4 bytes = 21.1 MB).
#define PAD_STATIC_SCRATCH_BYTES (size_t(32) << 20)

static __device__ __align__(256) unsigned char g_static_scratch[PAD_STATIC_SCRATCH_BYTES];

namespace pad {
namespace {

constexpr size_t kStaticScratchBytes = PAD_STATIC_SCRATCH_BYTES;

std::atomic<void *> g_scratch_addr[64];

// Device address of the array on the current device (set-up on first use).
pad_status static_scratch_address(void **out) {
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof msg, "cudaGetDevice: %s", cudaGetErrorString(e));
    set_last_error(msg);
    return PAD_ERR_CUDA;
  }
  if (device < 0 || device >= 64) {
    set_last_error("device ordinal out of range for the static scratch table");
    return PAD_ERR_UNSUPPORTED;
  }
  void *addr = g_scratch_addr[device].load(std::memory_order_acquire);
  if (addr == nullptr) {
    e = cudaGetSymbolAddress(&addr, g_static_scratch);
    if (e != cudaSuccess || addr == nullptr) {
      char msg[256];
      snprintf(msg, sizeof msg, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
      set_last_error(msg);
      return PAD_ERR_CUDA;
    }
    g_scratch_addr[device].store(addr, std::memory_order_release);
  }
  *out = addr;
  return PAD_OK;
}

}  // namespace
}  // namespace pad

extern "C" pad_status pad_decode_static_scratch(const pad_tensor *q, const pad_tensor *k_cache,
                                                const pad_tensor *v_cache, const pad_tensor *block_tables,
                                                const pad_tensor *seq_lens, float scale, int32_t num_splits,
                                                pad_tensor *out, pad_tensor *lse, void *stream) {
  // The array holds the control block (merge counters) first and the split
  // partials after it.  Reject shapes that do not fit before launching.
  size_t control = 0, need = 0;
  bool empty_batch = false;
  if (q != nullptr && k_cache != nullptr && block_tables != nullptr && q->ndim == 3 && k_cache->ndim == 4 &&
      block_tables->ndim == 2) {
    empty_batch = q->shape[0] == 0;
    const int32_t kv_dtype = k_cache->dtype == PAD_FP8_E4M3 ? PAD_FP8_E4M3 : PAD_BF16;
    pad_plan plan;
    if (pad_decode_plan_ex(q->shape[0], q->shape[1], k_cache->shape[1], q->shape[2], k_cache->shape[2],
                           block_tables->shape[1], num_splits, kv_dtype, -1, &plan) == PAD_OK) {
      control = (size_t)plan.control_bytes;
      need = control + (size_t)plan.workspace_bytes;
      if (need > pad::kStaticScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "this shape needs %zu bytes of split scratch; the static array holds %zu "
                 "(use fewer splits or pad_decode)",
                 need, pad::kStaticScratchBytes);
        pad::set_last_error(msg);
        return PAD_ERR_WORKSPACE;
      }
    }
  }
  // Only a launch that merges partitions touches the array: an empty batch or
  // one partition per sequence needs no address, and a malformed call is
  // rejected by the validation below before any buffer is looked at.
  void *scratch = nullptr;
  if (need > 0 && !empty_batch) {
    pad_status st = pad::static_scratch_address(&scratch);
    if (st != PAD_OK) return st;
  }
  char *partials = scratch != nullptr ? static_cast<char *>(scratch) + control : nullptr;
  const size_t partials_bytes = scratch != nullptr ? pad::kStaticScratchBytes - control : 0;
  // The control block must start at zero.  A completed call leaves it zero, but
  // the array outlives every call, so it is cleared on the stream after the
  // arguments are validated and before the launch.
  return pad::decode_with_buffers(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits, out, lse,
                                  partials, partials_bytes, scratch, scratch != nullptr ? control : 0,
                                  /*clear_control=*/true, static_cast<cudaStream_t>(stream));
}
