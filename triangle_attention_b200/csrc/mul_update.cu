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
// c is a multiple of 64 and R = N*N with N % 8 == 0). A tile of 64 positions x
// 64 channels passes through shared memory as [channel][position] bf16. On the
// position-major side a thread takes 16 channels (32 contiguous bytes, a whole
// sector) of one position per tensor; on the channel-major side 16 bytes (8
// positions), eight lanes covering 128 contiguous bytes. Both shared-memory
// passes are free of bank conflicts. Arithmetic and rounding are those of the
// kernels above.
constexpr int kT = 64;

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ uint16_t bits_of(float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t *>(&b);
}
__device__ __forceinline__ float from_bits(uint16_t v) {
  return __uint_as_float((uint32_t)v << 16);
}

// 16 bf16 (32 bytes at p) as floats
__device__ __forceinline__ void load16(const __nv_bfloat16 *p, float (&o)[16]) {
  const uint4 v0 = *reinterpret_cast<const uint4 *>(p);
  const uint4 v1 = *reinterpret_cast<const uint4 *>(p + 8);
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    o[2 * e] = __uint_as_float(w[e] << 16);
    o[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}
// 16 floats rounded to bf16 into 32 bytes at p (one 32-byte store)
__device__ __forceinline__ void store16(__nv_bfloat16 *p, const float (&v)[16]) {
  uint32_t w[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) w[e] = pack2(v[2 * e], v[2 * e + 1]);
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
// 8 bf16 (16 bytes) of a shared-memory row as a uint4
__device__ __forceinline__ void unpack8(const uint4 v, float (&o)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    o[2 * e] = __uint_as_float(w[e] << 16);
    o[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}

__global__ void __launch_bounds__(256) gate_in_fwd_tiled(const __nv_bfloat16 *__restrict__ pg,
                                                         int64_t R, int c, int64_t ldpg,
                                                         __nv_bfloat16 *__restrict__ a_cm,
                                                         __nv_bfloat16 *__restrict__ b_cm) {
  __shared__ __align__(16) uint16_t ta[kT][kT], tb[kT][kT];
  const int64_t p0 = (int64_t)blockIdx.x * kT;
  const int ch0 = blockIdx.y * kT;
  const int pl = threadIdx.x & (kT - 1), g = threadIdx.x / kT;   // position, 16-channel group
  const __nv_bfloat16 *row = pg + (p0 + pl) * ldpg + ch0 + 16 * g;
  {
    float ap[16], ag[16];
    load16(row, ap);
    load16(row + c, ag);
#pragma unroll
    for (int e = 0; e < 16; ++e) ta[16 * g + e][pl] = bits_of(sigm(ag[e]) * ap[e]);
  }
  {
    float bp[16], bg[16];
    load16(row + 2 * c, bp);
    load16(row + 3 * c, bg);
#pragma unroll
    for (int e = 0; e < 16; ++e) tb[16 * g + e][pl] = bits_of(sigm(bg[e]) * bp[e]);
  }
  __syncthreads();
  for (int it = threadIdx.x; it < 2 * kT * 8; it += 256) {
    const int tns = it / (kT * 8), chl = (it / 8) % kT, k = it % 8;
    const uint4 v = *reinterpret_cast<const uint4 *>(&(tns ? tb : ta)[chl][8 * k]);
    *reinterpret_cast<uint4 *>((tns ? b_cm : a_cm) + (int64_t)(ch0 + chl) * R + p0 + 8 * k) = v;
  }
}

__global__ void __launch_bounds__(256) gate_in_bwd_tiled(const __nv_bfloat16 *__restrict__ da_cm,
                                                         const __nv_bfloat16 *__restrict__ db_cm,
                                                         const __nv_bfloat16 *__restrict__ pg,
                                                         int64_t R, int c, int64_t ldpg,
                                                         __nv_bfloat16 *__restrict__ dpg) {
  __shared__ __align__(16) uint16_t ta[kT][kT], tb[kT][kT];
  const int64_t p0 = (int64_t)blockIdx.x * kT;
  const int ch0 = blockIdx.y * kT;
  for (int it = threadIdx.x; it < 2 * kT * 8; it += 256) {
    const int tns = it / (kT * 8), chl = (it / 8) % kT, k = it % 8;
    const uint4 v = *reinterpret_cast<const uint4 *>((tns ? db_cm : da_cm) +
                                                     (int64_t)(ch0 + chl) * R + p0 + 8 * k);
    *reinterpret_cast<uint4 *>(&(tns ? tb : ta)[chl][8 * k]) = v;
  }
  __syncthreads();
  const int pl = threadIdx.x & (kT - 1), g = threadIdx.x / kT;
  const int64_t off = (p0 + pl) * ldpg + ch0 + 16 * g;
  {
    float ap[16], ag[16], r0[16], r1[16];
    load16(pg + off, ap);
    load16(pg + off + c, ag);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float da = from_bits(ta[16 * g + e][pl]);
      const float sa = sigm(ag[e]);
      r0[e] = da * sa;
      r1[e] = da * ap[e] * sa * (1.0f - sa);
    }
    store16(dpg + off, r0);
    store16(dpg + off + c, r1);
  }
  {
    float bp[16], bg[16], r2[16], r3[16];
    load16(pg + off + 2 * c, bp);
    load16(pg + off + 3 * c, bg);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float db = from_bits(tb[16 * g + e][pl]);
      const float sb = sigm(bg[e]);
      r2[e] = db * sb;
      r3[e] = db * bp[e] * sb * (1.0f - sb);
    }
    store16(dpg + off + 2 * c, r2);
    store16(dpg + off + 3 * c, r3);
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

// colsum_strided_kernel with 8 columns per thread and 16 rows of 16-byte loads in
// flight; each column is still summed over the block's rows in row order, so
// the partial sums are bit-identical to the one-column-per-thread form.
__global__ void colsum_strided_vec(const __nv_bfloat16 *__restrict__ m, int64_t rows, int64_t ld,
                                   int cols, float *__restrict__ part) {
  const int64_t span = (rows + gridDim.x - 1) / gridDim.x;
  const int64_t r0 = (int64_t)blockIdx.x * span;
  const int64_t r1 = r0 + span < rows ? r0 + span : rows;
  const int col = threadIdx.x * 8;
  if (col >= cols) return;
  float s[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) s[e] = 0.0f;
  constexpr int kAhead = 16;
  int64_t r = r0;
  for (; r + kAhead <= r1; r += kAhead) {
    uint4 v[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u)
      v[u] = *reinterpret_cast<const uint4 *>(m + (r + u) * ld + col);
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      float x[8];
      unpack8(v[u], x);
#pragma unroll
      for (int e = 0; e < 8; ++e) s[e] += x[e];
    }
  }
  for (; r < r1; ++r) {
    float x[8];
    unpack8(*reinterpret_cast<const uint4 *>(m + r * ld + col), x);
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] += x[e];
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[(int64_t)blockIdx.x * cols + col + e] = s[e];
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
  if (tiled_shape(R, c) && ldpg % 16 == 0 && (reinterpret_cast<uintptr_t>(dpg) & 31) == 0 &&
      R / kT <= 0x7fffffffLL) {
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
  if (cols % 8 == 0 && ld % 8 == 0 && cols <= 8 * 1024) {
    const int threads = ((cols / 8 + 31) / 32) * 32;
    colsum_strided_vec<<<kProjBlocks, threads, 0, stream>>>(m, rows, ld, cols, part);
    return cudaGetLastError();
  }
  colsum_strided_kernel<<<kProjBlocks, 256, 0, stream>>>(m, rows, ld, cols, part);
  return cudaGetLastError();
}

}  // namespace tri
