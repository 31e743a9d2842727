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

// ------------------------------------------------ 64 x 64 tiled versions --
// For shapes whose both sides are multiples of 64 (every shape of the update:
// c is a multiple of 64 and R = N*N with N % 8 == 0). A tile moves through
// shared memory as [64 channels][32 position pairs] words, each word the bf16
// values of two consecutive positions: warp w reads (or writes) channels
// 8w .. 8w+7 of 64 positions with one 16-byte access per position, and the
// channel-major side moves 16 bytes (8 positions) per access, eight lanes
// covering 128 contiguous bytes. Both shared-memory passes are free of bank
// conflicts. Arithmetic and rounding are those of the kernels above.
constexpr int kT = 64;

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ float lo_of(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_of(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 8 bf16 of a uint4 as floats
__device__ __forceinline__ void unpack8(const uint4 v, float (&o)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    o[2 * e] = lo_of(w[e]);
    o[2 * e + 1] = hi_of(w[e]);
  }
}

__global__ void __launch_bounds__(256) gate_in_fwd_tiled(const __nv_bfloat16 *__restrict__ pg,
                                                         int64_t R, int c, int64_t ldpg,
                                                         __nv_bfloat16 *__restrict__ a_cm,
                                                         __nv_bfloat16 *__restrict__ b_cm) {
  __shared__ __align__(16) uint32_t ta[kT][kT / 2], tb[kT][kT / 2];
  const int64_t p0 = (int64_t)blockIdx.x * kT;
  const int ch0 = blockIdx.y * kT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cg = ch0 + warp * 8;
  float av[2][8], bv[2][8];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const __nv_bfloat16 *row = pg + (p0 + 2 * lane + k) * ldpg + cg;
    float ap[8], ag[8], bp[8], bg[8];
    unpack8(*reinterpret_cast<const uint4 *>(row), ap);
    unpack8(*reinterpret_cast<const uint4 *>(row + c), ag);
    unpack8(*reinterpret_cast<const uint4 *>(row + 2 * c), bp);
    unpack8(*reinterpret_cast<const uint4 *>(row + 3 * c), bg);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      av[k][e] = sigm(ag[e]) * ap[e];
      bv[k][e] = sigm(bg[e]) * bp[e];
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    ta[warp * 8 + e][lane] = pack2(av[0][e], av[1][e]);
    tb[warp * 8 + e][lane] = pack2(bv[0][e], bv[1][e]);
  }
  __syncthreads();
  for (int it = threadIdx.x; it < 2 * kT * 8; it += 256) {
    const int tns = it / (kT * 8), chl = (it / 8) % kT, k = it % 8;
    const uint4 v = *reinterpret_cast<const uint4 *>(&(tns ? tb : ta)[chl][4 * k]);
    *reinterpret_cast<uint4 *>((tns ? b_cm : a_cm) + (int64_t)(ch0 + chl) * R + p0 + 8 * k) = v;
  }
}

__global__ void __launch_bounds__(256) gate_in_bwd_tiled(const __nv_bfloat16 *__restrict__ da_cm,
                                                         const __nv_bfloat16 *__restrict__ db_cm,
                                                         const __nv_bfloat16 *__restrict__ pg,
                                                         int64_t R, int c, int64_t ldpg,
                                                         __nv_bfloat16 *__restrict__ dpg) {
  __shared__ __align__(16) uint32_t ta[kT][kT / 2], tb[kT][kT / 2];
  const int64_t p0 = (int64_t)blockIdx.x * kT;
  const int ch0 = blockIdx.y * kT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int it = threadIdx.x; it < 2 * kT * 8; it += 256) {
    const int tns = it / (kT * 8), chl = (it / 8) % kT, k = it % 8;
    const uint4 v = *reinterpret_cast<const uint4 *>((tns ? db_cm : da_cm) +
                                                     (int64_t)(ch0 + chl) * R + p0 + 8 * k);
    *reinterpret_cast<uint4 *>(&(tns ? tb : ta)[chl][4 * k]) = v;
  }
  __syncthreads();
  const int cg = ch0 + warp * 8;
  uint32_t dw[8], ew[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    dw[e] = ta[warp * 8 + e][lane];
    ew[e] = tb[warp * 8 + e][lane];
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int64_t off = (p0 + 2 * lane + k) * ldpg + cg;
    float ap[8], ag[8], bp[8], bg[8];
    unpack8(*reinterpret_cast<const uint4 *>(pg + off), ap);
    unpack8(*reinterpret_cast<const uint4 *>(pg + off + c), ag);
    unpack8(*reinterpret_cast<const uint4 *>(pg + off + 2 * c), bp);
    unpack8(*reinterpret_cast<const uint4 *>(pg + off + 3 * c), bg);
    uint32_t o0[4], o1[4], o2[4], o3[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float r0[2], r1[2], r2[2], r3[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float da = k ? hi_of(dw[e + u]) : lo_of(dw[e + u]);
        const float db = k ? hi_of(ew[e + u]) : lo_of(ew[e + u]);
        const float sa = sigm(ag[e + u]), sb = sigm(bg[e + u]);
        r0[u] = da * sa;
        r1[u] = da * ap[e + u] * sa * (1.0f - sa);
        r2[u] = db * sb;
        r3[u] = db * bp[e + u] * sb * (1.0f - sb);
      }
      o0[e / 2] = pack2(r0[0], r0[1]);
      o1[e / 2] = pack2(r1[0], r1[1]);
      o2[e / 2] = pack2(r2[0], r2[1]);
      o3[e / 2] = pack2(r3[0], r3[1]);
    }
    *reinterpret_cast<uint4 *>(dpg + off) = make_uint4(o0[0], o0[1], o0[2], o0[3]);
    *reinterpret_cast<uint4 *>(dpg + off + c) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
    *reinterpret_cast<uint4 *>(dpg + off + 2 * c) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
    *reinterpret_cast<uint4 *>(dpg + off + 3 * c) = make_uint4(o3[0], o3[1], o3[2], o3[3]);
  }
}

// out [cols][rows] = in [rows][cols]^T, both sides multiples of 64; the bits
// move unchanged (two rows' values of one column per shared-memory word).
__global__ void __launch_bounds__(256) transpose_tiled(const __nv_bfloat16 *__restrict__ in,
                                                       int64_t rows, int64_t cols,
                                                       __nv_bfloat16 *__restrict__ out) {
  __shared__ __align__(16) uint32_t t[kT][kT / 2];
  const int64_t col_tiles = cols / kT;
  const int64_t r0 = ((int64_t)blockIdx.x / col_tiles) * kT;
  const int64_t c0 = ((int64_t)blockIdx.x % col_tiles) * kT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __nv_bfloat16 *src = in + (r0 + 2 * lane) * cols + c0 + 8 * warp;
  const uint4 va = *reinterpret_cast<const uint4 *>(src);
  const uint4 vb = *reinterpret_cast<const uint4 *>(src + cols);
  const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
  for (int e = 0; e < 8; ++e)
    t[warp * 8 + e][lane] = __byte_perm(wa[e / 2], wb[e / 2], (e & 1) ? 0x7632 : 0x5410);
  __syncthreads();
  for (int it = threadIdx.x; it < kT * 8; it += 256) {
    const int chl = it / 8, k = it % 8;
    *reinterpret_cast<uint4 *>(out + (c0 + chl) * rows + r0 + 8 * k) =
        *reinterpret_cast<const uint4 *>(&t[chl][4 * k]);
  }
}

bool tiled_shape(int64_t a, int64_t b) { return a % kT == 0 && b % kT == 0; }

int blocks_for(int64_t n) {
  int64_t b = (n + 255) / 256;
  if (b > 148 * 16) b = 148 * 16;
  return (int)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_gate_in_fwd(const __nv_bfloat16 *pg, int64_t R, int c, int64_t ldpg,
                               __nv_bfloat16 *a_cm, __nv_bfloat16 *b_cm, cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  if (tiled_shape(R, c) && ldpg % 8 == 0 && R / kT <= 0x7fffffffLL) {
    gate_in_fwd_tiled<<<dim3((unsigned)(R / kT), c / kT), 256, 0, stream>>>(pg, R, c, ldpg, a_cm,
                                                                            b_cm);
    return cudaGetLastError();
  }
  dim3 grid((unsigned)((R + kTile - 1) / kTile), c / kTile);
  gate_in_fwd_kernel<<<grid, dim3(kTile, 8), 0, stream>>>(pg, R, c, ldpg, a_cm, b_cm);
  return cudaGetLastError();
}

cudaError_t launch_gate_in_bwd(const __nv_bfloat16 *da_cm, const __nv_bfloat16 *db_cm,
                               const __nv_bfloat16 *pg, int64_t R, int c, int64_t ldpg,
                               __nv_bfloat16 *dpg, cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  if (tiled_shape(R, c) && ldpg % 8 == 0 && R / kT <= 0x7fffffffLL) {
    gate_in_bwd_tiled<<<dim3((unsigned)(R / kT), c / kT), 256, 0, stream>>>(da_cm, db_cm, pg, R,
                                                                            c, ldpg, dpg);
    return cudaGetLastError();
  }
  dim3 grid((unsigned)((R + kTile - 1) / kTile), c / kTile);
  gate_in_bwd_kernel<<<grid, dim3(kTile, 8), 0, stream>>>(da_cm, db_cm, pg, R, c, ldpg, dpg);
  return cudaGetLastError();
}

cudaError_t launch_transpose(const __nv_bfloat16 *in, int64_t rows, int64_t cols,
                             __nv_bfloat16 *out, cudaStream_t stream) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  if (tiled_shape(rows, cols) && (rows / kT) * (cols / kT) <= 0x7fffffffLL) {
    transpose_tiled<<<(unsigned)((rows / kT) * (cols / kT)), 256, 0, stream>>>(in, rows, cols,
                                                                               out);
    return cudaGetLastError();
  }
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
