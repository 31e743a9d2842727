// Host-side interface of the triangle-multiplication kernels (trimul.cu).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace tri {

struct MulArgs {
  int N, C;
  __nv_bfloat16 *out;                // D of the product, channel-major [C][N][N]
  int32_t *status;
};

// D[c][m][n] = sum_k X[c](m, k) Y[c](n, k) for every channel. x_mn / y_mn: the
// operand's stored matrix has k as its rows (MN-major) instead of its columns
// (K-major). The maps come from encode_mul_operand with the same majors.
// d: the output stack, stored through 64 x 32 boxes (encode_mul_output).
cudaError_t launch_trimul_gemm(bool x_mn, bool y_mn, const CUtensorMap &x, const CUtensorMap &y,
                               const CUtensorMap &d, const MulArgs &args, cudaStream_t stream);

}  // namespace tri
