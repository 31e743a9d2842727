// Diagnostic: the bounded-wait path of the tcgen05 kernels, exercised on its
// own. One warp waits on an mbarrier that nothing ever arrives at, with the
// same wait primitive and limit as the forward and backward kernels; the wait
// gives up, the kernel records TRI_ATTN_ERR_TIMEOUT in the workspace status
// word and returns. No trap, no fault: the CUDA context stays usable.
#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"
#include "ptx.cuh"

namespace tri {
namespace {

__global__ void unsatisfied_wait_kernel(int32_t *status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // phase 0 of a barrier that expects one arrival and never gets it
  const bool done = mbar_wait(&bar, 0);
  if (!done && threadIdx.x == 0) report_status(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_unsatisfied_wait(int32_t *status, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), stream);
  if (e != cudaSuccess) return e;
  unsatisfied_wait_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace tri
