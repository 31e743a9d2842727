// Host-side interface of the LayerNorm / projection kernels (proj.cu).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace tri {

// Blocks of 256 threads of the row-parallel kernels (148 SMs x 4): the number
// of partial sums of every row reduction (one per block).
constexpr int kProjBlocks = 148 * 4;

struct ProjArgs {
  int64_t rows;                      // pair positions, all batch elements
  int64_t rows_per;                  // pair positions per batch element (bias layout)
  int cz, H;                         // channels of z (64, 128, 192, 256), bias heads (<= 8)
  float eps;
  const __nv_bfloat16 *z;            // [rows][cz]
  const float *gamma, *beta;         // [cz] (beta: forward only)
  const __nv_bfloat16 *w_b;          // [cz][H]
  __nv_bfloat16 *x;                  // LayerNorm output [rows][cz]: forward writes,
                                     // backward reads
  float *stats;                      // [rows][2]: mean, 1/sqrt(var + eps)
  __nv_bfloat16 *bias;               // forward: [batch][H][rows_per]
  const float *dx;                   // backward: gradient w.r.t. x from the projections
  const __nv_bfloat16 *dbias;        // backward: [batch][H][rows_per]
  __nv_bfloat16 *dz;                 // backward: [rows][cz]
  float *part;                       // backward: [kProjBlocks][cz * (2 + H)] partial sums
  int32_t *status;                   // backward: device status word (bounded waits)
};

int proj_partials();         // partial sums per row reduction (kProjBlocks)
cudaError_t launch_ln_fwd(const ProjArgs &a, cudaStream_t stream);
cudaError_t launch_ln_bwd(const ProjArgs &a, cudaStream_t stream);
// per-block partial column sums of m [rows][cols] into part [kProjBlocks][cols]
cudaError_t launch_colsum(const __nv_bfloat16 *m, int64_t rows, int cols, float *part,
                          cudaStream_t stream);
// One fixed-order sum over partials: out[(i / width) * out_stride + i % width] =
// sum_{k < n} part[k * part_stride + i], in k order, for i < len.
struct SumSeg {
  const float *part;
  int64_t n, part_stride, len;
  float *out;
  int64_t width, out_stride;
};
constexpr int kMaxSumSegs = 4;
struct SumSegs {
  SumSeg seg[kMaxSumSegs];
  int nseg;
  int64_t first_block[kMaxSumSegs];
};
cudaError_t launch_ordered_sum(const float *part, int64_t n, int64_t part_stride, int64_t len,
                               float *out, int64_t width, int64_t out_stride,
                               cudaStream_t stream);
// up to kMaxSumSegs sums in one launch
cudaError_t launch_ordered_sums(const SumSeg *segs, int nseg, cudaStream_t stream);

}  // namespace tri
