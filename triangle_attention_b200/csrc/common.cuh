// Shared definitions of the kernels: the problem in the variant frame, device
// status codes and the host-side launch entry points of each kernel file.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace tri {

// Device status codes (same values as tri_attn_status).
enum : int32_t { kStatusOk = 0, kStatusTimeout = 5, kStatusBounds = 6 };

// A problem seen from the variant's own frame: attention row r, query x, key y.
// Pair tensor element (r, x, h, cc) sits at r*sR + x*sX + h*c + cc; bias entry
// (h, x, y) at h*N*N + x*bX + y*bY; the key mask entry (r, y) at
// r*mask_stride + y.
struct Frame {
  int N, H, c;
  int variant;  // 0 starting node, 1 ending node
  int64_t sR, sX;
  int64_t bX, bY;
  const uint8_t *mask;
  int64_t mask_stride;
  int32_t *status;  // device status word, never null inside a launch
  // attention rows [row0, row_end) of the variant frame that this call computes:
  // rows of B stacked problems count on, row b*N + r being row r of problem b
  // (0 and B*N unless the caller asked for a row shard)
  int row0, row_end;
  int B;  // problems in the batch (the CUDA-core kernels take one at a time)
};

// Record a device-side failure (first writer wins; the value never goes back
// to zero inside a call).
__device__ __forceinline__ void report_status(int32_t *status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// Diagnostic kernel: a bounded wait that nothing satisfies (see selftest.cu).
cudaError_t launch_unsatisfied_wait(int32_t *status, cudaStream_t stream);
// Diagnostic kernel: tensor-core issue rate by instruction shape (see selftest.cu).
cudaError_t launch_mma_probe(int n, int layout, int ctas, int instructions,
                             unsigned long long *cycles, int32_t *status, cudaStream_t stream);
// Diagnostic kernel: both device exp2 evaluations of x[0..n) (see selftest.cu).
cudaError_t launch_exp2_eval(const float *x, float *y_fma, float *y_mufu, int64_t n,
                             cudaStream_t stream);

__host__ __device__ inline int64_t pair_elems(const Frame &f) {
  return (int64_t)f.N * f.N * f.H * f.c;
}

// ------------------------------------------------------- CUDA-core path --
// T = float (the fp32 path) or __nv_bfloat16 (bf16 shapes the tensor-core
// kernels do not take); arithmetic in fp32.
template <typename T>
cudaError_t launch_f32_fwd(const Frame &f, const T *q, const T *k, const T *v, const T *bias,
                           const T *gate, T *out, float *lse, cudaStream_t stream);

// Scratch of the fp32 backward, carved by the API layer.
struct F32BwdScratch {
  float *du;        // [N, N, H, c] compact, variant frame
  float *D;         // [N, H, N]
  float *part_dq;   // [ntile][N, N, H, c]
  float *part_dk;   // [ntile][N, N, H, c]
  float *part_dv;   // [ntile][N, N, H, c]
  float *part_db;   // [ngroups][H, N, N] (variant frame), only if ngroups > 1
  int ntile, ngroups;
};

int f32_bwd_tile();
void f32_bwd_plan(const Frame &f, int *ntile, int *ngroups);
template <typename T>
cudaError_t launch_f32_bwd(const Frame &f, const T *q, const T *k, const T *v, const T *bias,
                           const T *gate, const T *out, const float *lse, const T *dout, T *dq,
                           T *dk, T *dv, T *dbias, T *dgate, const F32BwdScratch &s,
                           cudaStream_t stream);

// ---------------------------------------------- fixed-order reductions (any) --
// out[r,x,h,cc] (storage position via the frame) = scale * sum_{t<nparts} part[t][...]
template <typename T>
cudaError_t launch_pair_reduce(const Frame &f, const float *part, int nparts, float scale,
                               T *out, cudaStream_t stream);
// dbias (storage layout) = sum_{g<ngroups} part[g][h][x][y] (variant frame)
template <typename T>
cudaError_t launch_bias_reduce(const Frame &f, const float *part, int ngroups, T *dbias,
                               cudaStream_t stream);

}  // namespace tri
