// Scratch memory for kvq_decode_attention_noalloc: decode attention for callers
// that cannot allocate device memory.
//
// The regular entry point asks its caller for a workspace (split-K partials and
// merge counters).  Some callers have no way to provide one: code that runs with
// an allocator-free runtime, a host that owns every byte of device memory through
// its own pool and cannot hand a slice to a library, or a loop that must never
// call cudaMalloc (it can synchronise the device).  For them the library keeps a
// fixed scratch array in device memory that exists as soon as the library is
// loaded (on every GPU that loads it, until the process exits).
//
// In host code the array's name is only a host-side stand-in for the device
// symbol; its device address is looked up once per device, with that device
// current, with cudaGetSymbolAddress, and that address is what the kernels get.
#include <mutex>

#include "kvq_internal.h"

namespace kvq {

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_mu;
void* g_ptr[64] = {};
}  // namespace

// Device address of the scratch array on `device`, which must be the current
// device (looked up on the first call per device).  Returns the CUDA error of the
// lookup, if any, or cudaErrorInvalidDevice when another device is current.
cudaError_t noalloc_scratch(int device, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != device || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return cudaSuccess;
}

}  // namespace kvq
