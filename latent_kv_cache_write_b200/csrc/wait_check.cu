// Diagnostic of the library's failure path.  One thread waits, with the bounded wait that
// every tensor-core kernel uses, on an mbarrier nothing arrives at.  The wait gives up
// after its limit (~2 s), records its site in the device error word and the kernel
// returns normally, so the host reads MLA_ERR_TIMEOUT from mla_device_error and the
// context stays usable.  Nothing faults, traps or hangs.
#include "launch.h"
#include "tc_ptx.cuh"

namespace mla {
namespace {

constexpr uint32_t WAIT_CHECK_SITE = 0x7FFu;

__global__ void wait_check_kernel(unsigned int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  // phase 0 of a fresh barrier completes only when one thread arrives: none does
  if (threadIdx.x == 0) tc::mbar_wait(&bar, 0, &abort, err, WAIT_CHECK_SITE, 0);
}

}  // namespace

cudaError_t wait_check(unsigned int* err, cudaStream_t st) {
  wait_check_kernel<<<1, 32, 0, st>>>(err);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace mla
