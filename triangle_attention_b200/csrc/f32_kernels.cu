// CUDA-core path of gated triangle self-attention (FFMA, no TF32): the fp32
// path, and the bf16 path for the shapes the tensor-core kernels do not take
// (head dimensions other than 32, N not a multiple of 8). The caller's tensors
// are of type T (float or bf16): every load widens to fp32, all arithmetic is
// fp32 and every result is rounded to T once. Also the fixed-order reductions
// that both dtypes use for their backward.
//
// Forward: one thread per query, online softmax over key tiles staged in
// shared memory, accurate expf/logf.
//
// Backward: each CTA owns one (query tile, key tile, head) block of the
// probability matrix and walks a group of attention rows in order. For every
// row it recomputes that block of probabilities once and uses it for all four
// gradients ("TurboPairFormer accelera fino a 1,73x l'addestramento di
// OpenFold3 nei test", section "Dove si impiega il tempo"): the pair-bias
// gradient stays in registers across the rows, while the dq/dk/dv
// contributions of the block are written as fp32 partials that a second
// kernel sums in a fixed order. Nothing is accumulated with atomics, so
// repeated calls give bit-identical results.
#include <cmath>
#include <cuda_bf16.h>

#include "common.cuh"

namespace tri {
namespace {

constexpr int kCMax = 64;     // largest head dimension of the fp32 path
constexpr int kFwdQ = 64;     // queries per CTA (one per thread)
constexpr int kFwdK = 32;     // keys per shared-memory tile
constexpr int kT = 32;        // backward block edge (queries and keys)
constexpr int kBwdThreads = 256;
constexpr int kEntries = kT * kT / kBwdThreads;  // probability entries per thread

__device__ __forceinline__ float ld(const float *p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
template <typename T> __device__ __forceinline__ T to_out(float x);
template <> __device__ __forceinline__ float to_out<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

template <typename T>
__global__ void __launch_bounds__(kFwdQ)
f32_fwd_kernel(Frame f, const T *__restrict__ q, const T *__restrict__ k,
               const T *__restrict__ v, const T *__restrict__ bias,
               const T *__restrict__ gate, T *__restrict__ out,
               float *__restrict__ lse) {
  __shared__ float ks[kFwdK][kCMax];
  __shared__ float vs[kFwdK][kCMax];
  __shared__ unsigned char keep[kFwdK];
  const int C = f.c, N = f.N;
  const int x = blockIdx.x * kFwdQ + threadIdx.x;
  const int h = blockIdx.y;
  const int r = blockIdx.z;
  const bool active = x < N;
  const float scale = 1.0f / sqrtf((float)C);
  const int64_t px = (int64_t)r * f.sR + (int64_t)x * f.sX + (int64_t)h * C;
  const int64_t hb = (int64_t)h * N * N;

  float qr[kCMax], acc[kCMax];
#pragma unroll
  for (int cc = 0; cc < kCMax; ++cc) {
    qr[cc] = (active && cc < C) ? ld(q + px + cc) : 0.0f;
    acc[cc] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;

  for (int y0 = 0; y0 < N; y0 += kFwdK) {
    __syncthreads();
    for (int e = threadIdx.x; e < kFwdK * C; e += kFwdQ) {
      const int yy = e / C, cc = e % C, y = y0 + yy;
      float kv = 0.0f, vv = 0.0f;
      if (y < N) {
        const int64_t py = (int64_t)r * f.sR + (int64_t)y * f.sX + (int64_t)h * C + cc;
        kv = ld(k + py);
        vv = ld(v + py);
      }
      ks[yy][cc] = kv;
      vs[yy][cc] = vv;
    }
    for (int yy = threadIdx.x; yy < kFwdK; yy += kFwdQ) {
      const int y = y0 + yy;
      keep[yy] = (y < N) && (!f.mask || f.mask[(int64_t)r * f.mask_stride + y] != 0);
    }
    __syncthreads();
    if (!active) continue;
    for (int yy = 0; yy < kFwdK; ++yy) {
      if (!keep[yy]) continue;
      const int y = y0 + yy;
      float dot = 0.0f;
#pragma unroll
      for (int cc = 0; cc < kCMax; ++cc)
        if (cc < C) dot = fmaf(qr[cc], ks[yy][cc], dot);
      const float s = dot * scale + ld(bias + hb + (int64_t)x * f.bX + (int64_t)y * f.bY);
      if (s > m) {
        const float a = expf(m - s);  // m = -inf gives 0
        l = l * a + 1.0f;
#pragma unroll
        for (int cc = 0; cc < kCMax; ++cc)
          if (cc < C) acc[cc] = fmaf(acc[cc], a, vs[yy][cc]);
        m = s;
      } else {
        const float p = expf(s - m);
        l += p;
#pragma unroll
        for (int cc = 0; cc < kCMax; ++cc)
          if (cc < C) acc[cc] = fmaf(p, vs[yy][cc], acc[cc]);
      }
    }
  }
  if (!active) return;
  const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
  for (int cc = 0; cc < kCMax; ++cc) {
    if (cc < C) {
      const float sg = 1.0f / (1.0f + expf(-ld(gate + px + cc)));
      out[px + cc] = to_out<T>(sg * (acc[cc] * inv));
    }
  }
  lse[((int64_t)r * f.H + h) * N + x] = l > 0.0f ? m + logf(l) : -INFINITY;
}

// du = dout * sigmoid(g) (compact, variant frame); D = sum_c dout * out;
// dgate = dout * out * (1 - sigmoid(g)).
template <typename T>
__global__ void f32_bwd_pre_kernel(Frame f, const T *__restrict__ gate,
                                   const T *__restrict__ out,
                                   const T *__restrict__ dout, float *__restrict__ du,
                                   float *__restrict__ D, T *__restrict__ dgate) {
  const int64_t total = (int64_t)f.N * f.N * f.H;
  const int C = f.c;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int h = (int)(w % f.H);
    const int64_t x = (w / f.H) % f.N;
    const int64_t r = w / ((int64_t)f.H * f.N);
    const int64_t px = r * f.sR + x * f.sX + (int64_t)h * C;
    const int64_t cx = w * C;
    float d = 0.0f;
    for (int cc = 0; cc < C; ++cc) {
      const float sg = 1.0f / (1.0f + expf(-ld(gate + px + cc)));
      const float go = ld(dout + px + cc), o = ld(out + px + cc);
      du[cx + cc] = go * sg;
      d = fmaf(go, o, d);
      dgate[px + cc] = to_out<T>(go * o * (1.0f - sg));
    }
    D[(r * f.H + h) * f.N + x] = d;
  }
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
f32_bwd_main_kernel(Frame f, const T *__restrict__ q, const T *__restrict__ k,
                    const T *__restrict__ v, const T *__restrict__ bias,
                    const float *__restrict__ lse, const float *__restrict__ du,
                    const float *__restrict__ Dv, float *__restrict__ part_dq,
                    float *__restrict__ part_dk, float *__restrict__ part_dv,
                    float *__restrict__ part_db, T *__restrict__ dbias, int ngroups,
                    int rows_per_group) {
  __shared__ float Qs[kT][kCMax + 1], Us[kT][kCMax + 1], Ks[kT][kCMax + 1], Vs[kT][kCMax + 1];
  __shared__ float Ps[kT][kT + 1], Ss[kT][kT + 1];
  __shared__ float lse_s[kT], D_s[kT];
  __shared__ unsigned char keep[kT];

  const int C = f.c, N = f.N, H = f.H;
  const int x0 = blockIdx.x * kT, y0 = blockIdx.y * kT;
  const int h = blockIdx.z % H, g = blockIdx.z / H;
  const int r0 = g * rows_per_group;
  const int r1 = min(N, r0 + rows_per_group);
  const float scale = 1.0f / sqrtf((float)C);
  const int64_t hb = (int64_t)h * N * N;
  const int64_t pair = (int64_t)N * N * H * C;

  float bval[kEntries], dbacc[kEntries];
#pragma unroll
  for (int i = 0; i < kEntries; ++i) {
    const int e = threadIdx.x + kBwdThreads * i;
    const int x = x0 + e / kT, y = y0 + e % kT;
    bval[i] = (x < N && y < N) ? ld(bias + hb + (int64_t)x * f.bX + (int64_t)y * f.bY) : 0.0f;
    dbacc[i] = 0.0f;
  }

  for (int r = r0; r < r1; ++r) {
    __syncthreads();
    for (int e = threadIdx.x; e < kT * C; e += kBwdThreads) {
      const int t = e / C, cc = e % C;
      const int x = x0 + t, y = y0 + t;
      float qv = 0.0f, uv = 0.0f, kv = 0.0f, vv = 0.0f;
      if (x < N) {
        qv = ld(q + (int64_t)r * f.sR + (int64_t)x * f.sX + (int64_t)h * C + cc);
        uv = du[(((int64_t)r * N + x) * H + h) * C + cc];
      }
      if (y < N) {
        const int64_t py = (int64_t)r * f.sR + (int64_t)y * f.sX + (int64_t)h * C + cc;
        kv = ld(k + py);
        vv = ld(v + py);
      }
      Qs[t][cc] = qv; Us[t][cc] = uv; Ks[t][cc] = kv; Vs[t][cc] = vv;
    }
    for (int t = threadIdx.x; t < kT; t += kBwdThreads) {
      const int x = x0 + t, y = y0 + t;
      lse_s[t] = x < N ? lse[((int64_t)r * H + h) * N + x] : -INFINITY;
      D_s[t] = x < N ? Dv[((int64_t)r * H + h) * N + x] : 0.0f;
      keep[t] = (y < N) && (!f.mask || f.mask[(int64_t)r * f.mask_stride + y] != 0);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kEntries; ++i) {
      const int e = threadIdx.x + kBwdThreads * i;
      const int xx = e / kT, yy = e % kT;
      float p = 0.0f, ds = 0.0f;
      const float L = lse_s[xx];
      if (keep[yy] && L > -INFINITY) {
        float dot = 0.0f, dp = 0.0f;
        for (int cc = 0; cc < C; ++cc) {
          dot = fmaf(Qs[xx][cc], Ks[yy][cc], dot);
          dp = fmaf(Us[xx][cc], Vs[yy][cc], dp);
        }
        p = expf(dot * scale + bval[i] - L);
        ds = p * (dp - D_s[xx]);
      }
      Ps[xx][yy] = p;
      Ss[xx][yy] = ds;
      dbacc[i] += ds;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kT * C; e += kBwdThreads) {
      const int t = e / C, cc = e % C;
      float aq = 0.0f, ak = 0.0f, av = 0.0f;
      for (int j = 0; j < kT; ++j) {
        aq = fmaf(Ss[t][j], Ks[j][cc], aq);   // dq_t  = sum_y ds[t][y] k[y]
        ak = fmaf(Ss[j][t], Qs[j][cc], ak);   // dk_t  = sum_x ds[x][t] q[x]
        av = fmaf(Ps[j][t], Us[j][cc], av);   // dv_t  = sum_x p[x][t] du[x]
      }
      const int x = x0 + t, y = y0 + t;
      if (x < N) part_dq[blockIdx.y * pair + (((int64_t)r * N + x) * H + h) * C + cc] = aq;
      if (y < N) {
        const int64_t o = blockIdx.x * pair + (((int64_t)r * N + y) * H + h) * C + cc;
        part_dk[o] = ak;
        part_dv[o] = av;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kEntries; ++i) {
    const int e = threadIdx.x + kBwdThreads * i;
    const int x = x0 + e / kT, y = y0 + e % kT;
    if (x >= N || y >= N) continue;
    if (ngroups == 1)
      dbias[hb + (int64_t)x * f.bX + (int64_t)y * f.bY] = to_out<T>(dbacc[i]);
    else
      part_db[((int64_t)g * H + h) * N * N + (int64_t)x * N + y] = dbacc[i];
  }
}

template <typename T>
__global__ void pair_reduce_kernel(Frame f, const float *__restrict__ part, int nparts,
                                   float scale, T *__restrict__ out) {
  const int64_t total = pair_elems(f);
  const int C = f.c;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int t = 0; t < nparts; ++t) s += part[t * total + w];
    const int cc = (int)(w % C);
    const int h = (int)((w / C) % f.H);
    const int64_t x = (w / ((int64_t)C * f.H)) % f.N;
    const int64_t r = w / ((int64_t)C * f.H * f.N);
    out[r * f.sR + x * f.sX + (int64_t)h * C + cc] = to_out<T>(s * scale);
  }
}

template <typename T>
__global__ void bias_reduce_kernel(Frame f, const float *__restrict__ part, int ngroups,
                                   T *__restrict__ dbias) {
  const int64_t nn = (int64_t)f.N * f.N;
  const int64_t total = nn * f.H;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int g = 0; g < ngroups; ++g) s += part[g * total + w];
    const int64_t h = w / nn, x = (w / f.N) % f.N, y = w % f.N;
    dbias[h * nn + x * f.bX + y * f.bY] = to_out<T>(s);
  }
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  if (b > 148 * 32) b = 148 * 32;
  return (int)(b < 1 ? 1 : b);
}

}  // namespace

template <typename T>
cudaError_t launch_f32_fwd(const Frame &f, const T *q, const T *k, const T *v, const T *bias,
                           const T *gate, T *out, float *lse, cudaStream_t stream) {
  if (f.N == 0) return cudaSuccess;
  dim3 grid((f.N + kFwdQ - 1) / kFwdQ, f.H, f.N);
  f32_fwd_kernel<T><<<grid, kFwdQ, 0, stream>>>(f, q, k, v, bias, gate, out, lse);
  return cudaGetLastError();
}

int f32_bwd_tile() { return kT; }

void f32_bwd_plan(const Frame &f, int *ntile, int *ngroups) {
  const int nt = (f.N + kT - 1) / kT;
  *ntile = nt;
  const int64_t tiles = (int64_t)nt * nt * f.H;
  int64_t g = (2 * 148 + tiles - 1) / (tiles > 0 ? tiles : 1);
  if (g < 1) g = 1;
  if (g > f.N) g = f.N > 0 ? f.N : 1;
  // equalise the group sizes
  const int rows = (int)((f.N + g - 1) / g);
  *ngroups = rows > 0 ? (f.N + rows - 1) / rows : 1;
}

template <typename T>
cudaError_t launch_f32_bwd(const Frame &f, const T *q, const T *k, const T *v, const T *bias,
                           const T *gate, const T *out, const float *lse, const T *dout, T *dq,
                           T *dk, T *dv, T *dbias, T *dgate, const F32BwdScratch &s,
                           cudaStream_t stream) {
  if (f.N == 0) return cudaSuccess;
  const int64_t rows_hx = (int64_t)f.N * f.N * f.H;
  f32_bwd_pre_kernel<T><<<grid_for(rows_hx, 256), 256, 0, stream>>>(f, gate, out, dout, s.du,
                                                                     s.D, dgate);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int rows_per_group = (f.N + s.ngroups - 1) / s.ngroups;
  dim3 grid(s.ntile, s.ntile, f.H * s.ngroups);
  f32_bwd_main_kernel<T><<<grid, kBwdThreads, 0, stream>>>(
      f, q, k, v, bias, lse, s.du, s.D, s.part_dq, s.part_dk, s.part_dv, s.part_db, dbias,
      s.ngroups, rows_per_group);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const float scale = 1.0f / sqrtf((float)f.c);
  if ((e = launch_pair_reduce<T>(f, s.part_dq, s.ntile, scale, dq, stream)) != cudaSuccess)
    return e;
  if ((e = launch_pair_reduce<T>(f, s.part_dk, s.ntile, scale, dk, stream)) != cudaSuccess)
    return e;
  if ((e = launch_pair_reduce<T>(f, s.part_dv, s.ntile, 1.0f, dv, stream)) != cudaSuccess)
    return e;
  if (s.ngroups > 1)
    return launch_bias_reduce<T>(f, s.part_db, s.ngroups, dbias, stream);
  return cudaSuccess;
}

template <typename T>
cudaError_t launch_pair_reduce(const Frame &f, const float *part, int nparts, float scale,
                               T *out, cudaStream_t stream) {
  const int64_t total = pair_elems(f);
  if (total == 0) return cudaSuccess;
  pair_reduce_kernel<T><<<grid_for(total, 256), 256, 0, stream>>>(f, part, nparts, scale, out);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bias_reduce(const Frame &f, const float *part, int ngroups, T *dbias,
                               cudaStream_t stream) {
  const int64_t total = (int64_t)f.N * f.N * f.H;
  if (total == 0) return cudaSuccess;
  bias_reduce_kernel<T><<<grid_for(total, 256), 256, 0, stream>>>(f, part, ngroups, dbias);
  return cudaGetLastError();
}

template cudaError_t launch_pair_reduce<float>(const Frame &, const float *, int, float, float *,
                                               cudaStream_t);
template cudaError_t launch_pair_reduce<__nv_bfloat16>(const Frame &, const float *, int, float,
                                                       __nv_bfloat16 *, cudaStream_t);
template cudaError_t launch_bias_reduce<float>(const Frame &, const float *, int, float *,
                                               cudaStream_t);
template cudaError_t launch_bias_reduce<__nv_bfloat16>(const Frame &, const float *, int,
                                                       __nv_bfloat16 *, cudaStream_t);
template cudaError_t launch_f32_fwd<float>(const Frame &, const float *, const float *,
                                           const float *, const float *, const float *, float *,
                                           float *, cudaStream_t);
template cudaError_t launch_f32_fwd<__nv_bfloat16>(const Frame &, const __nv_bfloat16 *,
                                                   const __nv_bfloat16 *, const __nv_bfloat16 *,
                                                   const __nv_bfloat16 *, const __nv_bfloat16 *,
                                                   __nv_bfloat16 *, float *, cudaStream_t);
template cudaError_t launch_f32_bwd<float>(const Frame &, const float *, const float *,
                                           const float *, const float *, const float *,
                                           const float *, const float *, const float *, float *,
                                           float *, float *, float *, float *,
                                           const F32BwdScratch &, cudaStream_t);
template cudaError_t launch_f32_bwd<__nv_bfloat16>(
    const Frame &, const __nv_bfloat16 *, const __nv_bfloat16 *, const __nv_bfloat16 *,
    const __nv_bfloat16 *, const __nv_bfloat16 *, const __nv_bfloat16 *, const float *,
    const __nv_bfloat16 *, __nv_bfloat16 *, __nv_bfloat16 *, __nv_bfloat16 *, __nv_bfloat16 *,
    __nv_bfloat16 *, const F32BwdScratch &, cudaStream_t);

}  // namespace tri
