// Host-side interface of the elementwise kernels of the triangle multiplicative
// update (mul_update.cu). R = pair positions; pg = [R][ldpg] pre-activations
// [ap | ag | bp | bg | gl] (bf16, biases included); a_cm, b_cm, da_cm, db_cm
// channel-major [c][R]. c and the channel counts are multiples of 32; ldpg and
// cz multiples of 8.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace tri {

cudaError_t launch_gate_in_fwd(const __nv_bfloat16 *pg, int64_t R, int c, int64_t ldpg,
                               __nv_bfloat16 *a_cm, __nv_bfloat16 *b_cm, cudaStream_t stream);
cudaError_t launch_gate_in_bwd(const __nv_bfloat16 *da_cm, const __nv_bfloat16 *db_cm,
                               const __nv_bfloat16 *pg, int64_t R, int c, int64_t ldpg,
                               __nv_bfloat16 *dpg, cudaStream_t stream);
// out [cols][rows] = in [rows][cols]^T
cudaError_t launch_transpose(const __nv_bfloat16 *in, int64_t rows, int64_t cols,
                             __nv_bfloat16 *out, cudaStream_t stream);
cudaError_t launch_out_fwd(const __nv_bfloat16 *pg, int64_t ldpg, int goff,
                           const __nv_bfloat16 *h, int64_t R, int cz, __nv_bfloat16 *y,
                           cudaStream_t stream);
cudaError_t launch_out_bwd(const __nv_bfloat16 *dy, const __nv_bfloat16 *pg, int64_t ldpg,
                           int goff, const __nv_bfloat16 *h, int64_t R, int cz,
                           __nv_bfloat16 *dh, __nv_bfloat16 *dpg, cudaStream_t stream);
// per-block column sums of the first `cols` columns of m [rows][ld] into
// part [kProjBlocks][cols] (fixed row order inside each block)
cudaError_t launch_colsum_strided(const __nv_bfloat16 *m, int64_t rows, int64_t ld, int cols,
                                  float *part, cudaStream_t stream);

}  // namespace tri
