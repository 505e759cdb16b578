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

// Device address of the array on the current device, looked up on the first
// call on each device with that device current.  Without -rdc the array lives
// in a module of its own; under CUDA's lazy module loading (the default since
// CUDA 12.2) this lookup is what loads that module and reserves the 32 MiB on
// the device, so it belongs in the first call, made before any stream capture.
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
  // Arguments are validated and the plan made exactly as for pad_decode (same
  // statuses, same order); then a shape whose control block and partials do
  // not fit the array is rejected, and every call that gets that far -- one
  // partition per sequence included -- looks up the array's address, so the
  // first such call on a device does the set-up.  The control block (merge
  // counters) sits at the array's start and is cleared on the stream before
  // the launch; the partials follow it.
  return pad::decode_with_scratch_array(q, k_cache, v_cache, block_tables, seq_lens, scale, num_splits, out, lse,
                                        pad::static_scratch_address, pad::kStaticScratchBytes,
                                        static_cast<cudaStream_t>(stream));
}
