// Self-test of the bounded device-side waits used by the tcgen05 kernels: one
// CTA waits on an mbarrier that nothing ever arrives at.  The wait must give up
// after `limit_us`, record MKA_ERR_DEVICE_TIMEOUT in the status word and let
// the kernel return normally, leaving the CUDA context usable.
#include "../../include/mka.h"
#include "kernels.h"
#include "sm100.cuh"

namespace mka {

__global__ void wait_timeout_kernel(unsigned long long limit_ns, int* status, int* result) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool done = sm100::mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
    *result = done ? 1 : 0;
  }
}

cudaError_t selftest_wait_timeout(int limit_us, int* status, int* result, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>((unsigned long long)limit_us * 1000ull, status, result);
  return cudaGetLastError();
}

}  // namespace mka
