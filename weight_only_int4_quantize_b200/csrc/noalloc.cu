// Fixed device scratch for awq_score_grid_static_scratch.
//
// The scratch lives in its own translation unit, and so in its own module of
// device code.  Under CUDA's lazy module loading (the default), the driver
// reserves it on a device only when this module is first used there, that
// is, by the set-up in the first awq_score_grid_static_scratch call on that
// device.  The library's other entry points never touch this module, so they
// do not pay for the reservation.
#include <cuda_runtime.h>

#include <mutex>

#include "w4.h"

namespace w4 {

__device__ __align__(256) unsigned char g_awq_static_scratch[W4_AWQ_STATIC_SCRATCH_BYTES];

// Address of the scratch on the current device.  It is looked up once per
// device, with that device current, and cached; every later call is a table
// read.  Returns the lookup's CUDA error, if any (nothing is cached then).
cudaError_t awq_static_scratch_address(void** ptr) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_awq_static_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

}  // namespace w4
