// Host-side interface of the tensor-core GEMM (gemm.cu).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace tri {

struct GemmArgs {
  int M, Nn, K, batch;               // D[batch][M][Nn] = X[batch](M x K) Y[batch](Nn x K)^T
  int nouts;                         // bf16 output tensors (1..4); fp32: 1
  int cols_per_out;                  // columns of D per bf16 output tensor (multiple of 64)
  int k_per_x;                       // K columns per X tensor map (multiple of 64): X may
                                     // be up to four tensors laid side by side along K
  int n_per_y, ny;                   // Y may be ny <= 4 tensors of n_per_y rows n each
                                     // (a multiple of 64 MN-major, of 128 K-major)
  int k_split;                       // > 0: split-K, batch index b sums K columns
                                     // [b*k_split, min(K, (b+1)*k_split)) of operands with no
                                     // batch dimension (multiple of 64); 0: a true batch
  const float *col_bias;             // bf16 outputs: col_bias[n - col_bias_from] is added to
  int col_bias_from;                 // column n >= col_bias_from before rounding (or null)
  int32_t *status;
};

// Operand maps. X: K columns [i*k_per_x, (i+1)*k_per_x) come from map i.
// Y: rows n in [i*n_per_y, (i+1)*n_per_y) come from map i (n_per_y = 0: one map).
struct GemmMaps {
  CUtensorMap map[4];
};

// Output tensor maps: bf16 outputs are stored through 64 x 32 boxes, the fp32
// output through 32 x 32 boxes.
struct GemmOuts {
  CUtensorMap map[4];
};

// x_mn / y_mn: the operand's stored matrix has k as its rows (MN-major) instead
// of its columns (K-major); the maps come with the matching boxes (64 x 128
// K-major, 64 x 64 MN-major).
cudaError_t launch_gemm_tc(bool x_mn, bool y_mn, bool f32_out, const GemmMaps &x,
                           const GemmMaps &y, const GemmOuts &d, const GemmArgs &args,
                           cudaStream_t stream);

}  // namespace tri
