// Failure detection without a GPU fault: a kernel whose bounded wait must give up.
//
// One block; its first thread waits, through the same bounded mbar_wait every kernel of the
// library uses, on an mbarrier that nothing ever completes.  After the wait limit the wait
// records bit 0 (a bounded wait gave up) in the device error word and returns false, and the
// kernel ends normally: no trap, no hang, the context stays usable.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fp8q {
namespace {

__global__ void k_selftest_wait(uint32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);     // expects one arrival; none is ever made
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0u, err);
}

}  // namespace

cudaError_t launch_selftest_wait(cudaStream_t st) {
  k_selftest_wait<<<1, 32, 0, st>>>(device_error_word());
  return cudaGetLastError();
}

}  // namespace fp8q
