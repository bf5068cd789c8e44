// Fixed device scratch for llattn_fwd_noalloc.
//
// The array lives in this translation unit alone, so its device memory is
// reserved only when this part of the library's device code is loaded on a
// device, which happens when llattn_fwd_noalloc first looks up its address
// there; programs that never call llattn_fwd_noalloc do not pay for it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/llattn.h"
#include "llattn_internal.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[LLATTN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

namespace llattn {

cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    // `dev` is current here, so this is the array's address on that device.
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace llattn
