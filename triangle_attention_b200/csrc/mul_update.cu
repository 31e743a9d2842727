// Elementwise kernels of the full triangle multiplicative update (the
// LayerNorms, the products and the contraction run on the projection and GEMM
// kernels). The update, per pair position p of the pair representation z:
//   [ap | ag | bp | bg | gl] = LayerNorm(z) W_in + b_in
//   a = sigmoid(ag) ap, b = sigmoid(bg) bp                (channel-major for
//   t = contraction of a and b over the third residue      the contraction)
//   y = sigmoid(gl) (LayerNorm_out(t) W_o + b_o)
// ("TurboPairFormer accelera fino a 1,73x l'addestramento di OpenFold3 nei
// test", section "Dove si impiega il tempo": triangle multiplication beside
// triangle attention in the pair stack). All arithmetic is fp32 on bf16 values;
// every result is rounded to bf16 once.
#include <cstdint>
#include <cuda_bf16.h>

#include "mul_update.cuh"
#include "proj.cuh"

namespace tri {
namespace {

constexpr int kTile = 32;

__device__ __forceinline__ float sigm(float v) { return 1.0f / (1.0f + __expf(-v)); }
__device__ __forceinline__ float f(const __nv_bfloat16 v) { return __bfloat162float(v); }

// a, b [c][R] from the pre-activations pg [R][ldpg] (columns ap 0.., ag c..,
// bp 2c.., bg 3c..): a 32-position x 32-channel tile goes through shared memory
// so both the reads (along channels) and the writes (along positions) are
// contiguous. Block 32 x 8 threads.
__global__ void gate_in_fwd_kernel(const __nv_bfloat16 *__restrict__ pg, int64_t R, int c,
                                   int64_t ldpg, __nv_bfloat16 *__restrict__ a_cm,
                                   __nv_bfloat16 *__restrict__ b_cm) {
  __shared__ float ta[kTile][kTile + 1], tb[kTile][kTile + 1];
  const int64_t p0 = (int64_t)blockIdx.x * kTile;
  const int ch0 = blockIdx.y * kTile;
  for (int i = threadIdx.y; i < kTile; i += blockDim.y) {
    const int64_t p = p0 + i;
    const int ch = ch0 + threadIdx.x;
    float av = 0.0f, bv = 0.0f;
    if (p < R) {
      const __nv_bfloat16 *row = pg + p * ldpg;
      av = sigm(f(row[c + ch])) * f(row[ch]);
      bv = sigm(f(row[3 * c + ch])) * f(row[2 * c + ch]);
    }
    ta[i][threadIdx.x] = av;
    tb[i][threadIdx.x] = bv;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < kTile; i += blockDim.y) {
    const int64_t p = p0 + threadIdx.x;
    const int ch = ch0 + i;
    if (p < R) {
      a_cm[(int64_t)ch * R + p] = __float2bfloat16_rn(ta[threadIdx.x][i]);
      b_cm[(int64_t)ch * R + p] = __float2bfloat16_rn(tb[threadIdx.x][i]);
    }
  }
}

// dpg columns 0 .. 4c of position p from da, db [c][R] (read through a shared
// tile) and the pre-activations: dap = da sigmoid(ag), dag = da ap s (1 - s).
__global__ void gate_in_bwd_kernel(const __nv_bfloat16 *__restrict__ da_cm,
                                   const __nv_bfloat16 *__restrict__ db_cm,
                                   const __nv_bfloat16 *__restrict__ pg, int64_t R, int c,
                                   int64_t ldpg, __nv_bfloat16 *__restrict__ dpg) {
  __shared__ float ta[kTile][kTile + 1], tb[kTile][kTile + 1];
  const int64_t p0 = (int64_t)blockIdx.x * kTile;
  const int ch0 = blockIdx.y * kTile;
  for (int i = threadIdx.y; i < kTile; i += blockDim.y) {
    const int64_t p = p0 + threadIdx.x;
    const int ch = ch0 + i;
    ta[threadIdx.x][i] = p < R ? f(da_cm[(int64_t)ch * R + p]) : 0.0f;
    tb[threadIdx.x][i] = p < R ? f(db_cm[(int64_t)ch * R + p]) : 0.0f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < kTile; i += blockDim.y) {
    const int64_t p = p0 + i;
    const int ch = ch0 + threadIdx.x;
    if (p >= R) continue;
    const __nv_bfloat16 *row = pg + p * ldpg;
    __nv_bfloat16 *drow = dpg + p * ldpg;
    const float da = ta[i][threadIdx.x], db = tb[i][threadIdx.x];
    const float ap = f(row[ch]), sa = sigm(f(row[c + ch]));
    const float bp = f(row[2 * c + ch]), sb = sigm(f(row[3 * c + ch]));
    drow[ch] = __float2bfloat16_rn(da * sa);
    drow[c + ch] = __float2bfloat16_rn(da * ap * sa * (1.0f - sa));
    drow[2 * c + ch] = __float2bfloat16_rn(db * sb);
    drow[3 * c + ch] = __float2bfloat16_rn(db * bp * sb * (1.0f - sb));
  }
}

// out [cols][rows] = in [rows][cols]^T through a 32 x 32 shared tile; block
// blockIdx.x is tile (blockIdx.x % col_tiles, blockIdx.x / col_tiles).
__global__ void transpose_kernel(const __nv_bfloat16 *__restrict__ in, int64_t rows,
                                 int64_t cols, __nv_bfloat16 *__restrict__ out) {
  __shared__ __nv_bfloat16 t[kTile][kTile + 2];
  const int64_t col_tiles = (cols + kTile - 1) / kTile;
  const int64_t r0 = ((int64_t)blockIdx.x / col_tiles) * kTile;
  const int64_t c0 = ((int64_t)blockIdx.x % col_tiles) * kTile;
  for (int i = threadIdx.y; i < kTile; i += blockDim.y) {
    const int64_t r = r0 + i, col = c0 + threadIdx.x;
    if (r < rows && col < cols) t[i][threadIdx.x] = in[r * cols + col];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < kTile; i += blockDim.y) {
    const int64_t col = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && col < cols) out[col * rows + r] = t[threadIdx.x][i];
  }
}

// y = sigmoid(gl) h, gl = pg[:, goff ..] (b_in already added), 8 channels per thread.
__global__ void out_fwd_kernel(const __nv_bfloat16 *__restrict__ pg, int64_t ldpg, int goff,
                               const __nv_bfloat16 *__restrict__ h, int64_t R, int cz,
                               __nv_bfloat16 *__restrict__ y) {
  const int64_t groups = R * cz / 8;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < groups;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = w / (cz / 8), ch = (w % (cz / 8)) * 8;
    const uint4 gv = *reinterpret_cast<const uint4 *>(pg + p * ldpg + goff + ch);
    const uint4 hv = *reinterpret_cast<const uint4 *>(h + p * cz + ch);
    const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&gv);
    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&hv);
    uint4 o;
    __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 gg = __bfloat1622float2(g2[e]), hh = __bfloat1622float2(h2[e]);
      o2[e] = __floats2bfloat162_rn(sigm(gg.x) * hh.x, sigm(gg.y) * hh.y);
    }
    *reinterpret_cast<uint4 *>(y + p * cz + ch) = o;
  }
}

// dh = dy sigmoid(gl); dgl = dy h s (1 - s) into dpg[:, goff ..].
__global__ void out_bwd_kernel(const __nv_bfloat16 *__restrict__ dy,
                               const __nv_bfloat16 *__restrict__ pg, int64_t ldpg, int goff,
                               const __nv_bfloat16 *__restrict__ h, int64_t R, int cz,
                               __nv_bfloat16 *__restrict__ dh, __nv_bfloat16 *__restrict__ dpg) {
  const int64_t groups = R * cz / 8;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < groups;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = w / (cz / 8), ch = (w % (cz / 8)) * 8;
    const uint4 dv = *reinterpret_cast<const uint4 *>(dy + p * cz + ch);
    const uint4 gv = *reinterpret_cast<const uint4 *>(pg + p * ldpg + goff + ch);
    const uint4 hv = *reinterpret_cast<const uint4 *>(h + p * cz + ch);
    const __nv_bfloat162 *d2 = reinterpret_cast<const __nv_bfloat162 *>(&dv);
    const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&gv);
    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&hv);
    uint4 o1, o2;
    __nv_bfloat162 *a2 = reinterpret_cast<__nv_bfloat162 *>(&o1);
    __nv_bfloat162 *b2 = reinterpret_cast<__nv_bfloat162 *>(&o2);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 dd = __bfloat1622float2(d2[e]), gg = __bfloat1622float2(g2[e]),
                   hh = __bfloat1622float2(h2[e]);
      const float sx = sigm(gg.x), sy = sigm(gg.y);
      a2[e] = __floats2bfloat162_rn(dd.x * sx, dd.y * sy);
      b2[e] = __floats2bfloat162_rn(dd.x * hh.x * sx * (1.0f - sx), dd.y * hh.y * sy * (1.0f - sy));
    }
    *reinterpret_cast<uint4 *>(dh + p * cz + ch) = o1;
    *reinterpret_cast<uint4 *>(dpg + p * ldpg + goff + ch) = o2;
  }
}

// Per-block column sums of m [rows][ld] (first `cols` columns) into
// part [kProjBlocks][cols]: block b takes the rows b*span .. in order, thread t
// the columns t, t + 256, ...
__global__ void colsum_strided_kernel(const __nv_bfloat16 *__restrict__ m, int64_t rows,
                                      int64_t ld, int cols, float *__restrict__ part) {
  const int64_t span = (rows + gridDim.x - 1) / gridDim.x;
  const int64_t r0 = (int64_t)blockIdx.x * span;
  const int64_t r1 = r0 + span < rows ? r0 + span : rows;
  for (int col = threadIdx.x; col < cols; col += blockDim.x) {
    float s = 0.0f;
    for (int64_t r = r0; r < r1; ++r) s += f(m[r * ld + col]);
    part[(int64_t)blockIdx.x * cols + col] = s;
  }
}

int blocks_for(int64_t n) {
  int64_t b = (n + 255) / 256;
  if (b > 148 * 16) b = 148 * 16;
  return (int)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_gate_in_fwd(const __nv_bfloat16 *pg, int64_t R, int c, int64_t ldpg,
                               __nv_bfloat16 *a_cm, __nv_bfloat16 *b_cm, cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  dim3 grid((unsigned)((R + kTile - 1) / kTile), c / kTile);
  gate_in_fwd_kernel<<<grid, dim3(kTile, 8), 0, stream>>>(pg, R, c, ldpg, a_cm, b_cm);
  return cudaGetLastError();
}

cudaError_t launch_gate_in_bwd(const __nv_bfloat16 *da_cm, const __nv_bfloat16 *db_cm,
                               const __nv_bfloat16 *pg, int64_t R, int c, int64_t ldpg,
                               __nv_bfloat16 *dpg, cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  dim3 grid((unsigned)((R + kTile - 1) / kTile), c / kTile);
  gate_in_bwd_kernel<<<grid, dim3(kTile, 8), 0, stream>>>(da_cm, db_cm, pg, R, c, ldpg, dpg);
  return cudaGetLastError();
}

cudaError_t launch_transpose(const __nv_bfloat16 *in, int64_t rows, int64_t cols,
                             __nv_bfloat16 *out, cudaStream_t stream) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  const int64_t tiles = ((cols + kTile - 1) / kTile) * ((rows + kTile - 1) / kTile);
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  transpose_kernel<<<(unsigned)tiles, dim3(kTile, 8), 0, stream>>>(in, rows, cols, out);
  return cudaGetLastError();
}

cudaError_t launch_out_fwd(const __nv_bfloat16 *pg, int64_t ldpg, int goff,
                           const __nv_bfloat16 *h, int64_t R, int cz, __nv_bfloat16 *y,
                           cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  out_fwd_kernel<<<blocks_for(R * cz / 8), 256, 0, stream>>>(pg, ldpg, goff, h, R, cz, y);
  return cudaGetLastError();
}

cudaError_t launch_out_bwd(const __nv_bfloat16 *dy, const __nv_bfloat16 *pg, int64_t ldpg,
                           int goff, const __nv_bfloat16 *h, int64_t R, int cz,
                           __nv_bfloat16 *dh, __nv_bfloat16 *dpg, cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  out_bwd_kernel<<<blocks_for(R * cz / 8), 256, 0, stream>>>(dy, pg, ldpg, goff, h, R, cz, dh,
                                                              dpg);
  return cudaGetLastError();
}

cudaError_t launch_colsum_strided(const __nv_bfloat16 *m, int64_t rows, int64_t ld, int cols,
                                  float *part, cudaStream_t stream) {
  colsum_strided_kernel<<<kProjBlocks, 256, 0, stream>>>(m, rows, ld, cols, part);
  return cudaGetLastError();
}

}  // namespace tri
