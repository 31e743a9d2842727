// Diagnostics. The bounded-wait path of the tcgen05 kernels, exercised on its
// own; the forward's two exp2 evaluations (MUFU ex2.approx and the FMA-pipe
// polynomial) over caller-given exponents, for their error tests; and the issue
// rate of the tensor-core instruction shapes the kernels use.
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

// One CTA per SM: a single thread issues `instructions` (rounded up to a
// multiple of 8) tcgen05.mma (M = 128,
// K = 16, bf16 operands of zeros, fp32 accumulator) into one accumulator back to
// back, then waits (bounded) for their completion; cycles[cta] = SM clock cycles
// from the first issue to the completion. LAYOUT 0: A [128][32] and B [N][32]
// K-major with the 64-byte swizzle; LAYOUT 1: A and B MN-major (A 128-byte, B
// 64-byte swizzle); LAYOUT 2: A from tensor memory (columns 256..), B MN-major
// with the 64-byte swizzle (the forward's O += P V form).
constexpr uint32_t kProbeOperandBytes = 48 * 1024;
template <int N, int LAYOUT>
__global__ void __launch_bounds__(128, 1) mma_probe_kernel(int instructions,
                                                           unsigned long long *cycles,
                                                           int32_t *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *done = reinterpret_cast<uint64_t *>(smem + kProbeOperandBytes);
  uint32_t *tmem_base = reinterpret_cast<uint32_t *>(smem + kProbeOperandBytes + 8);
  for (uint32_t i = threadIdx.x; i < kProbeOperandBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    tmem_alloc(tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base;
  if (threadIdx.x == 0) {
    fence_proxy_async_smem();
    const uint32_t a = smem_u32(smem), b = smem_u32(smem + 32768);
    const uint32_t id = make_idesc_bf16(128, N, LAYOUT == 1, LAYOUT >= 1);
    // descriptors of the eight K steps computed once, so the issuing thread
    // spends as little as possible between instructions
    uint64_t da[8], db[8];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      // A within the first 32 KB (or tensor memory), B within the next 16 KB
      da[ks] = LAYOUT == 0 ? make_sdesc(a + (ks & 1) * 32, 16, 512, kSwizzle64B)
                           : make_sdesc(a + ks * 2048, 16384, 1024, kSwizzle128B);
      db[ks] = LAYOUT == 0 ? make_sdesc(b + (ks & 1) * 32, 16, 512, kSwizzle64B)
                           : make_sdesc(b + ks * 1024, 512, 512, kSwizzle64B);
    }
    const int rounds = (instructions + 7) / 8;
    const unsigned long long t0 = clock64();
    for (int r = 0; r < rounds; ++r) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        if (LAYOUT == 2)
          mma_ts(tmem, tmem + 256 + ks * 8, db[ks], id, (r | ks) ? 1u : 0u);
        else
          mma_ss(tmem, da[ks], db[ks], id, (r | ks) ? 1u : 0u);
      }
    }
    mma_commit(done);
    const bool ok = mbar_wait(done, 0);
    cycles[blockIdx.x] = clock64() - t0;
    if (!ok) report_status(status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int N, int LAYOUT>
cudaError_t launch_mma_probe_shape(int ctas, int instructions, unsigned long long *cycles,
                                   int32_t *status, cudaStream_t stream) {
  constexpr uint32_t smem = kProbeOperandBytes + 1024 + 1024;
  cudaError_t e = cudaFuncSetAttribute(mma_probe_kernel<N, LAYOUT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  mma_probe_kernel<N, LAYOUT><<<ctas, 128, smem, stream>>>(instructions, cycles, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mma_probe(int n, int layout, int ctas, int instructions,
                             unsigned long long *cycles, int32_t *status, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), stream);
  if (e != cudaSuccess) return e;
  if (layout == 1) return launch_mma_probe_shape<32, 1>(ctas, instructions, cycles, status, stream);
  if (layout == 2) return launch_mma_probe_shape<32, 2>(ctas, instructions, cycles, status, stream);
  switch (n) {
    case 32: return launch_mma_probe_shape<32, 0>(ctas, instructions, cycles, status, stream);
    case 64: return launch_mma_probe_shape<64, 0>(ctas, instructions, cycles, status, stream);
    case 128: return launch_mma_probe_shape<128, 0>(ctas, instructions, cycles, status, stream);
    default: return launch_mma_probe_shape<256, 0>(ctas, instructions, cycles, status, stream);
  }
}

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
