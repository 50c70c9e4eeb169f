// Fixed device scratch for mla_attend_fixed_scratch: the split-key partials of the
// attention kernel in a static device array instead of a caller workspace.  It lives in
// its own translation unit.  Under lazy module loading (the CUDA 12 default) the array
// takes device memory on a device only once the module is first used there; under eager
// loading (CUDA_MODULE_LOADING=EAGER) every context that loads the library holds it.
#include "launch.h"

#include <mutex>

namespace mla {
namespace {

static __device__ __align__(256) unsigned char g_attend_scratch[MLA_FIXED_SCRATCH_BYTES];

}  // namespace

cudaError_t fixed_scratch(void** ptr) {
  // One lookup per device, made with that device current: the symbol's address
  // differs between devices.
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attend_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

}  // namespace mla
