// Diagnostics. The bounded-wait path of the tcgen05 kernels, exercised on its
// own; and the forward's two exp2 evaluations (MUFU ex2.approx and the FMA-pipe
// polynomial) over caller-given exponents, for their error tests.
//
// Bounded wait: One warp waits on an mbarrier that nothing ever arrives at, with the
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

__global__ void exp2_eval_kernel(const float *__restrict__ x, float *__restrict__ y_fma,
                                 float *__restrict__ y_mufu, int64_t n) {
  for (int64_t i = 2 * (blockIdx.x * (int64_t)blockDim.x + threadIdx.x); i < n;
       i += 2 * (int64_t)gridDim.x * blockDim.x) {
    const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.0f;
    const float2 p = f2unpack(exp2_fma2(f2pack(x0, x1)));
    y_fma[i] = p.x;
    y_mufu[i] = ex2_approx(x0);
    if (i + 1 < n) {
      y_fma[i + 1] = p.y;
      y_mufu[i + 1] = ex2_approx(x1);
    }
  }
}

}  // namespace

cudaError_t launch_exp2_eval(const float *x, float *y_fma, float *y_mufu, int64_t n,
                             cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n / 2 + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  exp2_eval_kernel<<<(int)(blocks < 1 ? 1 : blocks), 256, 0, stream>>>(x, y_fma, y_mufu, n);
  return cudaGetLastError();
}

cudaError_t launch_unsatisfied_wait(int32_t *status, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), stream);
  if (e != cudaSuccess) return e;
  unsatisfied_wait_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace tri
