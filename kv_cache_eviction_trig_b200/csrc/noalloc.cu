// tria_prune_noalloc: the prune step with its scratch in a fixed device array
// owned by the library, for callers that cannot allocate device memory.
//
// Who needs it: a serving engine that reserves all device memory at start-up
// (one KV pool, one activation arena) and forbids allocation inside its decode
// loop, or a host callback that must not enter the CUDA allocator.  There,
// cudaMalloc and cudaFree are unavailable: they may fail once the pool owns
// the memory, and cudaFree waits for the whole device, which stalls a
// pipelined decode step.  Such a caller passes only the problem's inputs and
// outputs; the intermediate buffers (folded phasors, per-head raw scores,
// per-tile partial sums, selection lists, error word) live in the array below.
//
// The array is a file-scope device variable.  The library is compiled one
// translation unit per device module, and CUDA loads a module lazily, on first
// use: the array's device memory is therefore reserved by the first call on
// each device (the cudaGetSymbolAddress below loads the module), and every
// device that has made a call holds TRIA_NOALLOC_SCRATCH_BYTES of it until the
// process exits.  A caller that reserves all of a device's memory up front must
// make one call on that device before doing so (and before any stream capture);
// after that first call nothing is ever allocated again.  In host code the
// array's name only identifies the variable; its device address comes from
// cudaGetSymbolAddress, called with the device current.  Only a successful
// lookup is kept: a failed one (for example under memory pressure) is retried
// by the next call.  Every call on a device shares the array and finds the
// previous call's contents there: the call clears the error word; the other
// parts that must start at zero (the fused prune kernel's synchronisation words
// and histograms) start zero with the array and every prune leaves them zero;
// everything else is written before it is read.  Two calls whose kernels overlap on a
// device race on the array.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "tria.h"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[TRIA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

std::mutex g_lock;
void *g_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (nullptr on failure;
// the next call tries again).
void *scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> hold(g_lock);
  if (!g_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess) {
      g_ptr[dev] = p;
    } else {
      (void)cudaGetLastError();  // leave no sticky error for the caller's next CUDA call
    }
  }
  return g_ptr[dev];
}

}  // namespace

extern "C" tria_status tria_prune_noalloc(const tria_config *cfg, const tria_stats *stats,
                                          const tria_cache *cache, int32_t *sel_out,
                                          int32_t *device_error, void *stream) {
  size_t need = 0;
  tria_status s = tria_workspace_size(cfg, cache, &need);
  if (s != TRIA_OK) return s;
  if (need > (size_t)TRIA_NOALLOC_SCRATCH_BYTES) return TRIA_ERR_UNSUPPORTED;
  if (device_error && reinterpret_cast<uintptr_t>(device_error) % 4 != 0)
    return TRIA_ERR_INVALID_ARG;
  void *scratch = scratch_on_current_device();
  if (!scratch) return TRIA_ERR_CUDA;
  const size_t bytes = TRIA_NOALLOC_SCRATCH_BYTES;
  // only the error word needs clearing: the rest of the array's zero-at-rest prefix
  // (synchronisation words, histograms) starts zero and every prune leaves it zero
  if (cudaMemsetAsync(scratch, 0, 256, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TRIA_ERR_CUDA;
  if ((s = tria_prune(cfg, stats, cache, sel_out, scratch, bytes, stream)) != TRIA_OK) return s;
  if (device_error &&
      cudaMemcpyAsync(device_error, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TRIA_ERR_CUDA;
  return TRIA_OK;
}
