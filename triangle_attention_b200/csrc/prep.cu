// Preparation kernels of the bf16 path: key-mask bit packing, the transposed
// bias of the ending-node variant, and the backward preprocess that turns
// (dout, out, gate) into dU, D and dgate.
#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>

#include "bf16.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace tri {
namespace {

int blocks_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  if (b > 148 * 64) b = 148 * 64;
  return (int)(b < 1 ? 1 : b);
}

// One word = 32 keys of one row of the mask; bit j set when key 32*w + j exists
// and takes part. The mask's rows are N bytes apart: one per attention row of
// every problem (a per-row mask) or one per problem. Also resets the call's
// status word.
__global__ void mask_bits_kernel(Frame f, uint32_t *__restrict__ bits, int64_t rows,
                                 int64_t words_per_row, int32_t *status,
                                 int32_t *__restrict__ zero, int64_t nzero) {
  if (blockIdx.x == 0 && threadIdx.x == 0 && status) *status = kStatusOk;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < nzero;
       w += (int64_t)gridDim.x * blockDim.x)
    zero[w] = 0;
  const int64_t total = rows * words_per_row;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = w / words_per_row;
    const int64_t y0 = (w % words_per_row) * 32;
    uint32_t b = 0;
    for (int j = 0; j < 32; ++j) {
      const int64_t y = y0 + j;
      if (y < f.N && (!f.mask || f.mask[r * f.N + y] != 0)) b |= 1u << j;
    }
    bits[w] = b;
  }
}

__global__ void bias_transpose_kernel(const __nv_bfloat16 *__restrict__ in,
                                      __nv_bfloat16 *__restrict__ out, int N) {
  __shared__ __nv_bfloat16 t[32][33];
  const int64_t hb = (int64_t)blockIdx.z * N * N;
  const int bx = blockIdx.x * 32, by = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int row = by + i, col = bx + threadIdx.x;
    if (row < N && col < N) t[i][threadIdx.x] = in[hb + (int64_t)row * N + col];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int row = bx + i, col = by + threadIdx.x;
    if (row < N && col < N) out[hb + (int64_t)row * N + col] = t[threadIdx.x][i];
  }
}

__device__ __forceinline__ float sigmoid_fast(float g) {
  return rcp_approx(1.0f + ex2_approx(-g * 1.4426950408889634f));
}

// One thread per 8 channels (16 bytes) of one (problem p, storage row a, storage
// column b, head h), so a warp reads 512 contiguous bytes of each tensor per
// load; the four threads of one (p, a, b, h) sum their parts of D with two
// shuffles. Rows r of problem p count as attention row p*N + r of the batch.
__global__ void bwd_pre_bf16_kernel(Frame f, const __nv_bfloat16 *__restrict__ gate,
                                    const __nv_bfloat16 *__restrict__ out,
                                    const __nv_bfloat16 *__restrict__ out_res,
                                    const __nv_bfloat16 *__restrict__ dout,
                                    __nv_bfloat16 *__restrict__ du, float *__restrict__ D,
                                    __nv_bfloat16 *__restrict__ dgate,
                                    const float *__restrict__ lse, float *__restrict__ LD,
                                    int ending) {
  const int64_t total = (int64_t)f.B * f.N * f.N * f.H * 4;
  const unsigned group = 0xfu << (threadIdx.x & 28);   // the 4 lanes of one (a, b, h)
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int q = (int)(w & 3);                                // channels 8q .. 8q+7
    const int64_t e = w >> 2;                                  // (p, a, b, h)
    // one 64-bit division for the storage row p*N + a; the rest in 32 bits
    const int64_t pa = e / ((int64_t)f.H * f.N);              // p*N + a
    const uint32_t rem = (uint32_t)(e - pa * ((int64_t)f.H * f.N));   // b*H + h
    const int h = (int)(rem % (uint32_t)f.H);
    const int64_t b = rem / (uint32_t)f.H;
    const uint32_t pp = (uint32_t)pa / (uint32_t)f.N;          // B*N <= 2^16
    const int64_t aa = (uint32_t)pa - pp * (uint32_t)f.N;
    const int64_t r = pa - aa + (ending ? b : aa);             // row of the batch
    const int64_t x = ending ? aa : b;
    if (r < f.row0 || r >= f.row_end) continue;      // another call's row shard
    const int64_t so = w * 8;                                  // storage offset
    const int64_t co = (((r * f.N + x) * f.H) + h) * 32 + q * 8;   // compact variant frame
    const uint4 g4 = *reinterpret_cast<const uint4 *>(gate + so);
    const uint4 o4 = *reinterpret_cast<const uint4 *>(out + so);
    const uint4 d4 = *reinterpret_cast<const uint4 *>(dout + so);
    const uint4 r4 = out_res ? *reinterpret_cast<const uint4 *>(out_res + so)
                             : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
    const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w};
    const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w};
    const uint32_t rs[4] = {r4.x, r4.y, r4.z, r4.w};
    uint32_t uw[4], rw[4];
    float d = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float s0 = sigmoid_fast(bf16lo(gw[k])), s1 = sigmoid_fast(bf16hi(gw[k]));
      const float d0 = bf16lo(dw[k]), d1 = bf16hi(dw[k]);
      // the forward's fp32 output, as far as out and its residual carry it
      const float o0 = bf16lo(ow[k]) + bf16lo(rs[k]), o1 = bf16hi(ow[k]) + bf16hi(rs[k]);
      d = fmaf(d0, o0, d);
      d = fmaf(d1, o1, d);
      uw[k] = pack_bf16(d0 * s0, d1 * s1);
      rw[k] = pack_bf16(d0 * o0 * (1.0f - s0), d1 * o1 * (1.0f - s1));
    }
    *reinterpret_cast<uint4 *>(du + co) = make_uint4(uw[0], uw[1], uw[2], uw[3]);
    *reinterpret_cast<uint4 *>(dgate + so) = make_uint4(rw[0], rw[1], rw[2], rw[3]);
    // fixed combination order: (q0 + q1) + (q2 + q3)
    d += __shfl_xor_sync(group, d, 1);
    d += __shfl_xor_sync(group, d, 2);
    if (q == 0) {
      const int64_t rx = (r * f.H + h) * f.N + x;
      if (LD) {
        // (-lse*log2e of the query pair, -D of the pair) in one 16-byte group
        const float l = lse[rx];
        float *p = LD + ((r * f.H + h) * (f.N / 2) + (x >> 1)) * 4 + (x & 1);
        p[0] = l == -INFINITY ? -INFINITY : -l * 1.4426950408889634f;
        p[2] = -d;
      } else {
        D[rx] = d;
      }
    }
  }
}

// One thread per 8 channels of one contribution row: consecutive threads read
// consecutive 16-byte groups of the [tile][row][H][2][N][16] contributions; the
// nb tiles are summed in tile order in fp32, scaled and rounded once.
__global__ void partial_reduce_bf16_kernel(Frame f, const __nv_bfloat16 *__restrict__ pq,
                                           const __nv_bfloat16 *__restrict__ pk,
                                           const __nv_bfloat16 *__restrict__ pv, int nb,
                                           float scale, __nv_bfloat16 *__restrict__ dq,
                                           __nv_bfloat16 *__restrict__ dk,
                                           __nv_bfloat16 *__restrict__ dv) {
  const int64_t pair = (int64_t)f.N * f.N * f.H * 32;          // one problem
  const int64_t tile = pair * f.B;                               // one tile's contributions
  // 16-byte groups per attention row of one tensor and tile; rows (of the
  // batch) are outermost, so this call's row shard is one contiguous range
  const int64_t per_row = (int64_t)f.N * f.H * 4;
  const int64_t first = (int64_t)f.row0 * per_row;
  const int64_t per = (int64_t)(f.row_end - f.row0) * per_row;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < 3 * per;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int which = (int)(w / per);
    const int64_t gidx = first + (w - which * per);
    const __nv_bfloat16 *src = (which == 0 ? pq : which == 1 ? pk : pv) + gidx * 8;
    const float sc = which == 2 ? 1.0f : scale;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    // kBatch contributions in flight per thread, then added in tile order
    constexpr int kBatch = 8;
    for (int t0 = 0; t0 < nb; t0 += kBatch) {
      uint4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (t0 + u < nb) v[u] = __ldcs(reinterpret_cast<const uint4 *>(src + (t0 + u) * tile));
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (t0 + u >= nb) break;
        const uint32_t vw[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += bf16lo(vw[e]);
          acc[2 * e + 1] += bf16hi(vw[e]);
        }
      }
    }
    // gidx -> (r, h, half, i, c8) of the [r][H][2][N][16] layout
    // one 64-bit division for the row; the rest (below N*2*H <= 2^29) in 32 bits
    const int c8 = (int)(gidx & 1);
    const int64_t row_pieces = (int64_t)f.N * 2 * f.H;
    const int64_t r = (gidx >> 1) / row_pieces;
    const uint32_t rem = (uint32_t)((gidx >> 1) - r * row_pieces);
    const int64_t i = rem % (uint32_t)f.N;
    const int half = (int)((rem / (uint32_t)f.N) & 1u);
    const int h = (int)(rem / (2u * (uint32_t)f.N));
    const int64_t p = (uint32_t)r / (uint32_t)f.N;                // problem of row r
    __nv_bfloat16 *dst = (which == 0 ? dq : which == 1 ? dk : dv) + p * pair +
                         (r - p * f.N) * f.sR + i * f.sX + (int64_t)h * 32 + half * 16 + c8 * 8;
    *reinterpret_cast<uint4 *>(dst) =
        make_uint4(pack_bf16(acc[0] * sc, acc[1] * sc), pack_bf16(acc[2] * sc, acc[3] * sc),
                   pack_bf16(acc[4] * sc, acc[5] * sc), pack_bf16(acc[6] * sc, acc[7] * sc));
  }
}

}  // namespace

cudaError_t launch_partial_reduce_bf16(const Frame &f, const __nv_bfloat16 *part_q,
                                       const __nv_bfloat16 *part_k, const __nv_bfloat16 *part_v,
                                       int nb, float scale, __nv_bfloat16 *dq, __nv_bfloat16 *dk,
                                       __nv_bfloat16 *dv, cudaStream_t stream) {
  const int64_t work = 3 * ((int64_t)(f.row_end - f.row0) * f.N * f.H * 4);
  if (work <= 0) return cudaSuccess;
  partial_reduce_bf16_kernel<<<blocks_for(work, 256), 256, 0, stream>>>(f, part_q, part_k, part_v,
                                                                         nb, scale, dq, dk, dv);
  return cudaGetLastError();
}

cudaError_t launch_mask_bits(const Frame &f, uint32_t *bits, int64_t rows, int64_t words_per_row,
                             int32_t *status, int32_t *zero, int64_t nzero, cudaStream_t stream) {
  const int64_t work = rows * words_per_row > nzero ? rows * words_per_row : nzero;
  mask_bits_kernel<<<blocks_for(work, 256), 256, 0, stream>>>(f, bits, rows, words_per_row,
                                                              status, zero, nzero);
  return cudaGetLastError();
}

cudaError_t launch_bias_transpose(const __nv_bfloat16 *bias, __nv_bfloat16 *biasT, int N, int H,
                                  cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  dim3 grid((N + 31) / 32, (N + 31) / 32, H);
  bias_transpose_kernel<<<grid, dim3(32, 8), 0, stream>>>(bias, biasT, N);
  return cudaGetLastError();
}

cudaError_t launch_bwd_pre_bf16(const Frame &f, const __nv_bfloat16 *gate,
                                const __nv_bfloat16 *out, const __nv_bfloat16 *out_res,
                                const __nv_bfloat16 *dout,
                                __nv_bfloat16 *du, float *D, __nv_bfloat16 *dgate,
                                const float *lse, float *LD, cudaStream_t stream) {
  const int64_t total = (int64_t)f.B * f.N * f.N * f.H * 4;
  if (total == 0) return cudaSuccess;
  const int ending = f.variant == 1 ? 1 : 0;
  bwd_pre_bf16_kernel<<<blocks_for(total, 256), 256, 0, stream>>>(f, gate, out, out_res, dout,
                                                                  du, D, dgate, lse, LD, ending);
  return cudaGetLastError();
}

}  // namespace tri
