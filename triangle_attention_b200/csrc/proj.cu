// LayerNorm of the pair representation and the small projections around the
// attention's input projections (the large ones run on the tensor cores, see
// gemm.cu). The pages put LayerNorm at 14% of AlphaFold training time, at 10%
// of its theoretical speed before optimisation ("알파폴드 초기 학습 시간을
// 10시간으로 단축하는 ScaleFold", Stats), and fuse the gated attention with its
// projections ("HelixFold: An Efficient Implementation of AlphaFold2 using
// PaddlePaddle", proposed methods).
//
// One warp per pair position (row of z [rows][cz]); lane l holds channels
// l*CPL .. l*CPL + CPL - 1, so a warp reads and writes whole rows contiguously.
// Reductions over rows (dgamma, dbeta, the bias weights, the gate bias) are
// accumulated per warp over a fixed set of rows, added over a block's warps in
// warp order into one partial per block, and the partials are summed in block
// order by ordered_sum_kernel: repeated calls are bit-identical.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "ptx.cuh"
#include "proj.cuh"

namespace tri {
namespace {

constexpr int kMaxHeads = 8;
constexpr int kRowsPerWarp = 4;      // rows whose loads a warp keeps in flight

__device__ __forceinline__ float bf16_round(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// bias and dbias are [batch][H][rows_per]: entry (h, row) sits at
// bias_base(row) + h * rows_per (rows < 2^31, so 32-bit division suffices)
__device__ __forceinline__ int64_t bias_base(const ProjArgs &a, int64_t row) {
  const uint32_t b = (uint32_t)row / (uint32_t)a.rows_per;
  return row + (int64_t)b * (a.H - 1) * a.rows_per;
}

// CPL consecutive bf16 channels of one row, packed in pairs: one vector load
// of 4 to 16 bytes per lane.
template <int CPL>
__device__ __forceinline__ void load_raw(const __nv_bfloat16 *p, uint32_t (&w)[CPL / 2]) {
  if constexpr (CPL == 8) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
  } else if constexpr (CPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    w[0] = u.x, w[1] = u.y;
  } else {
#pragma unroll
    for (int e = 0; e < CPL / 2; ++e) w[e] = reinterpret_cast<const uint32_t *>(p)[e];
  }
}

template <int CPL>
__device__ __forceinline__ void unpack(const uint32_t (&w)[CPL / 2], float (&v)[CPL]) {
#pragma unroll
  for (int e = 0; e < CPL / 2; ++e) {
    v[2 * e] = bf16lo(w[e]);
    v[2 * e + 1] = bf16hi(w[e]);
  }
}

template <int CPL>
__device__ __forceinline__ void load_row(const __nv_bfloat16 *p, float (&v)[CPL]) {
  uint32_t w[CPL / 2];
  load_raw<CPL>(p, w);
  unpack<CPL>(w, v);
}

template <int CPL>
__device__ __forceinline__ void store_row(__nv_bfloat16 *p, const float (&v)[CPL]) {
  uint32_t w[CPL / 2];
#pragma unroll
  for (int e = 0; e < CPL / 2; ++e) w[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
  if constexpr (CPL == 8) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (CPL == 4) {
    *reinterpret_cast<uint2 *>(p) = make_uint2(w[0], w[1]);
  } else {
#pragma unroll
    for (int e = 0; e < CPL / 2; ++e) reinterpret_cast<uint32_t *>(p)[e] = w[e];
  }
}

template <int CPL>
__device__ __forceinline__ void load_row_f32(const float *p, float (&v)[CPL]) {
  if constexpr (CPL % 4 == 0) {
#pragma unroll
    for (int e = 0; e < CPL; e += 4) {
      const float4 u = *reinterpret_cast<const float4 *>(p + e);
      v[e] = u.x, v[e + 1] = u.y, v[e + 2] = u.z, v[e + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < CPL; e += 2) {
      const float2 u = *reinterpret_cast<const float2 *>(p + e);
      v[e] = u.x, v[e + 1] = u.y;
    }
  }
}

__host__ __device__ constexpr int ilog2(int n) { return n <= 1 ? 0 : 1 + ilog2(n / 2); }

// Warp sum of NV values at once (NV a power of two, at most 32) by recursive
// halving: at lane offsets 16, 8, ... each lane keeps half of its values and
// adds its partner's copy of that half, then the single value left is summed
// over the remaining offsets. NV - 1 + 5 - log2(NV) shuffles instead of 5 NV.
// Lane l returns the total of value l >> (5 - log2 NV); the order of the
// additions is fixed, so the result does not depend on scheduling.
template <int NV>
__device__ __forceinline__ float reduce_scatter(float (&v)[NV], int lane) {
  constexpr int L = ilog2(NV);
  static_assert((1 << L) == NV && NV <= 32, "NV must be a power of two <= 32");
#pragma unroll
  for (int st = 0, n = NV; st < L; ++st, n >>= 1) {
    const int off = 16 >> st;
    const bool upper = lane & off;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float keep = upper ? v[j + n / 2] : v[j];
      const float send = upper ? v[j] : v[j + n / 2];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float t = v[0];
#pragma unroll
  for (int off = 16 >> L; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
  return t;
}

// This lane's rows of w_b [cz][H] (channels c0 .. c0 + CPL - 1), zero past H.
template <int CPL, int HM>
__device__ __forceinline__ void load_wb(const ProjArgs &a, int c0, float (&wb)[CPL][HM]) {
#pragma unroll
  for (int e = 0; e < CPL; ++e)
#pragma unroll
    for (int h = 0; h < HM; ++h)
      wb[e][h] = h < a.H ? __bfloat162float(a.w_b[(c0 + e) * a.H + h]) : 0.0f;
}

// Rows are taken in groups of RPW by the warps in turn: group g goes to warp
// g mod (number of warps). A warp loads its next group while it works on the
// current one.
__device__ __forceinline__ int64_t first_group() {
  return blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
}
__device__ __forceinline__ int64_t group_stride() { return (int64_t)gridDim.x * (blockDim.x >> 5); }

template <int CPL, int RPW>
__device__ __forceinline__ void load_group(const __nv_bfloat16 *m, int64_t rows, int cols,
                                           int64_t r0, int c0, uint32_t (&w)[RPW][CPL / 2]) {
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    if (r0 + r < rows) {
      load_raw<CPL>(m + (r0 + r) * cols + c0, w[r]);
    } else {
#pragma unroll
      for (int e = 0; e < CPL / 2; ++e) w[r][e] = 0u;
    }
  }
}

// x = LayerNorm(z) * gamma + beta (bf16), stats = (mean, rstd), and
// bias[h][row] = sum_c x[c] w_b[c][h] from the rounded x the GEMM also reads.
// One warp per row, four rows at a time: the row sums of the four rows, then
// the 4 x HM bias dot products, are each one recursive-halving warp sum.
template <int CPL, int HM>
__global__ void __launch_bounds__(256, CPL <= 4 ? 3 : 2) ln_fwd_kernel(ProjArgs a) {
  constexpr int R = kRowsPerWarp;
  const int lane = threadIdx.x & 31;
  const int c0 = lane * CPL;
  const float inv_cz = 1.0f / a.cz;
  float wb[CPL][HM];
  load_wb<CPL, HM>(a, c0, wb);
  float g[CPL], bt[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) {
    g[e] = a.gamma[c0 + e];
    bt[e] = a.beta[c0 + e];
  }
  const int64_t groups = (a.rows + R - 1) / R;
  int64_t grp = first_group();
  uint32_t raw[R][CPL / 2];
  if (grp < groups) load_group<CPL, R>(a.z, a.rows, a.cz, grp * R, c0, raw);
  for (; grp < groups; grp += group_stride()) {
    const int64_t r0 = grp * R;
    float v[R][CPL];
#pragma unroll
    for (int r = 0; r < R; ++r) unpack<CPL>(raw[r], v[r]);
    if (grp + group_stride() < groups)
      load_group<CPL, R>(a.z, a.rows, a.cz, (grp + group_stride()) * R, c0, raw);
    float t[R], mean[R], rstd[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      t[r] = 0.0f;
#pragma unroll
      for (int e = 0; e < CPL; ++e) t[r] += v[r][e];
    }
    float tot = reduce_scatter<R>(t, lane);
#pragma unroll
    for (int r = 0; r < R; ++r) mean[r] = __shfl_sync(0xffffffffu, tot, r << (5 - ilog2(R))) * inv_cz;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      t[r] = 0.0f;
#pragma unroll
      for (int e = 0; e < CPL; ++e) t[r] += (v[r][e] - mean[r]) * (v[r][e] - mean[r]);
    }
    tot = reduce_scatter<R>(t, lane);
#pragma unroll
    for (int r = 0; r < R; ++r)
      rstd[r] = rsqrtf(__shfl_sync(0xffffffffu, tot, r << (5 - ilog2(R))) * inv_cz + a.eps);
    float sm = 0.0f, sr = 0.0f;                    // lane r < R writes row r's statistics
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int e = 0; e < CPL; ++e) v[r][e] = bf16_round((v[r][e] - mean[r]) * rstd[r] * g[e] + bt[e]);
      if (r0 + r < a.rows) store_row<CPL>(a.x + (r0 + r) * a.cz + c0, v[r]);
      if (lane == r) sm = mean[r], sr = rstd[r];
    }
    if (lane < R && r0 + lane < a.rows)
      reinterpret_cast<float2 *>(a.stats)[r0 + lane] = make_float2(sm, sr);
    float d[R * HM];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < HM; ++h) {
        float acc = 0.0f;
#pragma unroll
        for (int e = 0; e < CPL; ++e) acc += v[r][e] * wb[e][h];
        d[r * HM + h] = acc;
      }
    // lane l holds the total of (row, head) number l >> (5 - log2(R HM))
    constexpr int kShift = 5 - ilog2(R * HM);
    const float bsum = reduce_scatter<R * HM>(d, lane);
    const int idx = lane >> kShift, r = idx / HM, h = idx % HM;
    if ((lane & ((1 << kShift) - 1)) == 0 && h < a.H && r0 + r < a.rows)
      a.bias[bias_base(a, r0 + r) + h * a.rows_per] = __float2bfloat16_rn(bsum);
  }
}

// Backward staging: chunks of kChunkRows rows of z, x (bf16) and dx (fp32)
// come into shared memory by 1-D bulk copies, kBwdStages chunks in flight per
// block, so the warps never wait on single-row loads.
constexpr int kChunkRows = 32;                  // 4 rows per warp of a 256-thread block
constexpr int kBwdStages = 3;
constexpr uint32_t kAccBytes = 256 * (2 + kMaxHeads) * 4;

__host__ __device__ constexpr uint32_t bwd_stage_bytes(int cz) { return kChunkRows * cz * 8; }
__host__ __device__ constexpr uint32_t bwd_smem_bytes(int cz) {
  return kAccBytes + 128 + kBwdStages * bwd_stage_bytes(cz);
}

// Bounded wait on a staging barrier; false once it ran out or the block gave up.
__device__ __forceinline__ bool stage_wait(uint64_t *bar, uint32_t parity,
                                           volatile uint32_t *abort_flag, int32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t polls = 1; polls < kWaitMaxPolls; ++polls) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((polls & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
    }
  }
  *abort_flag = 1u;
  report_status(status, kStatusTimeout);
  return false;
}

// dz from dx (the projections' gradient w.r.t. x, fp32) plus the bias term
// sum_h dbias[h][row] w_b[c][h]; partial sums of dgamma, dbeta and
// dw_b[c][h] = sum_rows x[c] dbias[h][row] (x as the forward stored it), one
// set per block: each warp accumulates its rows, then the block's warps are
// added in warp order. Block b takes the chunks b, b + gridDim.x, ...; warp w
// the rows 4w .. 4w + 3 of each.
template <int CPL, int HM>
__global__ void __launch_bounds__(256) ln_bwd_kernel(ProjArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  float *acc = reinterpret_cast<float *>(smem);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kAccBytes);
  uint64_t *empty = full + kBwdStages;
  volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(empty + kBwdStages);
  uint8_t *stages = smem + kAccBytes + 128;
  const uint32_t stage_bytes = bwd_stage_bytes(a.cz);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c0 = lane * CPL;
  const float inv_cz = 1.0f / a.cz;
  const int64_t nchunks = (a.rows + kChunkRows - 1) / kChunkRows;
  const bool producer = threadIdx.x == 0;
  if (producer) {
    for (int st = 0; st < kBwdStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], blockDim.x >> 5);
    }
    *abort_flag = 0u;
    fence_barrier_init();
  }
  __syncthreads();

  // chunk `chunk` into stage st: z | x | dx of its rows
  auto issue = [&](int64_t chunk, int st) {
    const int64_t r0 = chunk * kChunkRows;
    const int64_t nr = a.rows - r0 < kChunkRows ? a.rows - r0 : (int64_t)kChunkRows;
    const uint32_t b16 = (uint32_t)(nr * a.cz * 2);
    uint8_t *dst = stages + st * stage_bytes;
    mbar_arrive_expect_tx(&full[st], 4 * b16);
    bulk_load(dst, a.z + r0 * a.cz, b16, &full[st]);
    bulk_load(dst + kChunkRows * a.cz * 2, a.x + r0 * a.cz, b16, &full[st]);
    bulk_load(dst + kChunkRows * a.cz * 4, a.dx + r0 * a.cz, 2 * b16, &full[st]);
  };
  int64_t issued = 0;                           // chunks of this block issued so far
  if (producer)
    for (int64_t ch = blockIdx.x; issued < kBwdStages - 1 && ch < nchunks; ch += gridDim.x)
      issue(ch, (int)(issued++));

  float wb[CPL][HM];
  load_wb<CPL, HM>(a, c0, wb);
  float g[CPL], dg[CPL], db[CPL], dwb[CPL][HM];
#pragma unroll
  for (int e = 0; e < CPL; ++e) {
    g[e] = a.gamma[c0 + e];
    dg[e] = db[e] = 0.0f;
#pragma unroll
    for (int h = 0; h < HM; ++h) dwb[e][h] = 0.0f;
  }
  int64_t i = 0;                                // chunks of this block consumed so far
  for (int64_t chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x, ++i) {
    const int st = (int)(i % kBwdStages);
    if (producer) {
      const int64_t next = chunk + (int64_t)(kBwdStages - 1) * gridDim.x;
      if (next < nchunks) {
        const int ns = (int)(issued % kBwdStages);
        // that stage last held chunk number issued - kBwdStages of this block
        const bool ok = issued < kBwdStages ||
                        stage_wait(&empty[ns], ((issued - kBwdStages) / kBwdStages) & 1,
                                   abort_flag, a.status);
        if (ok) issue(next, ns), ++issued;
      }
    }
    __syncwarp();
    // lane l fetches the statistics and dbias of row l of the chunk while the
    // chunk lands; the rows' threads take them by shuffle
    float2 lst = make_float2(0.0f, 0.0f);
    float ldb[HM];
    {
      const int64_t lrow = chunk * kChunkRows + lane;
      const bool in = lrow < a.rows;
      if (in) lst = reinterpret_cast<const float2 *>(a.stats)[lrow];
      const __nv_bfloat16 *dbias = a.dbias + (in ? bias_base(a, lrow) : 0);
#pragma unroll
      for (int h = 0; h < HM; ++h)
        ldb[h] = (in && h < a.H) ? __bfloat162float(dbias[h * a.rows_per]) : 0.0f;
    }
    if (!__all_sync(0xffffffffu,
                    stage_wait(&full[st], (i / kBwdStages) & 1, abort_flag, a.status)))
      break;
    const uint8_t *sz = stages + st * stage_bytes;
    const uint8_t *sx = sz + kChunkRows * a.cz * 2;
    const float *sdx = reinterpret_cast<const float *>(sz + kChunkRows * a.cz * 4);
    const int64_t r0 = chunk * kChunkRows + warp * 4;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int64_t row = r0 + r;
      if (row >= a.rows) break;                 // warp-uniform
      const int lr = warp * 4 + r;              // row within the chunk
      float z[CPL], x[CPL], u[CPL], xh[CPL];
      load_row<CPL>(reinterpret_cast<const __nv_bfloat16 *>(sz) + lr * a.cz + c0, z);
      load_row<CPL>(reinterpret_cast<const __nv_bfloat16 *>(sx) + lr * a.cz + c0, x);
      load_row_f32<CPL>(sdx + lr * a.cz + c0, u);
      const float2 stt = make_float2(__shfl_sync(0xffffffffu, lst.x, lr),
                                     __shfl_sync(0xffffffffu, lst.y, lr));
      float dbh[HM];
#pragma unroll
      for (int h = 0; h < HM; ++h) dbh[h] = __shfl_sync(0xffffffffu, ldb[h], lr);
      float s[2] = {0.0f, 0.0f};
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
#pragma unroll
        for (int h = 0; h < HM; ++h) {
          u[e] += dbh[h] * wb[e][h];
          dwb[e][h] += x[e] * dbh[h];
        }
        xh[e] = (z[e] - stt.x) * stt.y;
        dg[e] += u[e] * xh[e];
        db[e] += u[e];
        u[e] *= g[e];                           // dL/dxhat
        s[0] += u[e];
        s[1] += u[e] * xh[e];
      }
      const float tot = reduce_scatter<2>(s, lane);
      const float m1 = __shfl_sync(0xffffffffu, tot, 0) * inv_cz;
      const float m2 = __shfl_sync(0xffffffffu, tot, 16) * inv_cz;
#pragma unroll
      for (int e = 0; e < CPL; ++e) u[e] = stt.y * (u[e] - m1 - xh[e] * m2);
      store_row<CPL>(a.dz + row * a.cz + c0, u);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  __syncthreads();
  // copies issued but never consumed (only after a timeout) must land before exit
  if (producer)
    for (int64_t j = i; j < issued; ++j)
      mbar_wait(&full[j % kBwdStages], (j / kBwdStages) & 1);
  // block partials [dgamma cz | dbeta cz | dw_b cz*H], warps added in order
  const int len = a.cz * (2 + a.H);
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    if (warp == w) {
#pragma unroll
      for (int e = 0; e < CPL; ++e) {
        float *p0 = &acc[c0 + e], *p1 = &acc[a.cz + c0 + e];
        *p0 = (w ? *p0 : 0.0f) + dg[e];
        *p1 = (w ? *p1 : 0.0f) + db[e];
#pragma unroll
        for (int h = 0; h < HM; ++h)
          if (h < a.H) {
            float *p2 = &acc[2 * a.cz + (c0 + e) * a.H + h];
            *p2 = (w ? *p2 : 0.0f) + dwb[e][h];
          }
      }
    }
    __syncthreads();
  }
  float *part = a.part + blockIdx.x * (int64_t)len;
  for (int j = threadIdx.x; j < len; j += blockDim.x) part[j] = acc[j];
}

// Per-warp partial column sums of a [rows][cols] bf16 matrix (cols = 32*CPL),
// added per block in warp order: one partial row per block.
template <int CPL>
__global__ void __launch_bounds__(256) colsum_kernel(const __nv_bfloat16 *m, int64_t rows,
                                                     int cols, float *part) {
  __shared__ float acc[256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c0 = lane * CPL;
  float s[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) s[e] = 0.0f;
  const int64_t groups = (rows + kRowsPerWarp - 1) / kRowsPerWarp;
  for (int64_t grp = first_group(); grp < groups; grp += group_stride()) {
    const int64_t r0 = grp * kRowsPerWarp;
    float v[kRowsPerWarp][CPL];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
      if (r0 + r < rows) load_row<CPL>(m + (r0 + r) * cols + c0, v[r]);
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
      if (r0 + r < rows)
#pragma unroll
        for (int e = 0; e < CPL; ++e) s[e] += v[r][e];
  }
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    if (warp == w)
#pragma unroll
      for (int e = 0; e < CPL; ++e) acc[c0 + e] = (w ? acc[c0 + e] : 0.0f) + s[e];
    __syncthreads();
  }
  for (int i = threadIdx.x; i < cols; i += blockDim.x) part[blockIdx.x * (int64_t)cols + i] = acc[i];
}

// Each segment: out[i] = sum over k < n of part[k * part_stride + i], element i
// landing at out + (i / width) * out_stride + i % width. A block of 32 warps
// takes 32 consecutive elements of one segment (one per lane); warp w adds the
// k of its fixed share [w n / 32, (w + 1) n / 32) in order, then the 32 warp
// sums are added in warp order, so the result does not depend on scheduling.
// Several segments share one launch (blocks first_block[s] .. of segment s).
__global__ void __launch_bounds__(1024) ordered_sum_kernel(const __grid_constant__ SumSegs ss) {
  __shared__ float ws[32][33];
  int si = 0;
  while (si + 1 < ss.nseg && (int64_t)blockIdx.x >= ss.first_block[si + 1]) ++si;
  const SumSeg &g = ss.seg[si];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t i = ((int64_t)blockIdx.x - ss.first_block[si]) * 32 + lane;
  const int64_t k0 = warp * g.n / 32, k1 = (warp + 1) * g.n / 32;
  float s = 0.0f;
  if (i < g.len) {
    const float *p = g.part + i;
    int64_t k = k0;
    for (; k + 4 <= k1; k += 4) {
      const float v0 = p[k * g.part_stride], v1 = p[(k + 1) * g.part_stride];
      const float v2 = p[(k + 2) * g.part_stride], v3 = p[(k + 3) * g.part_stride];
      s += v0;
      s += v1;
      s += v2;
      s += v3;
    }
    for (; k < k1; ++k) s += p[k * g.part_stride];
  }
  ws[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && i < g.len) {
    float t = 0.0f;
    for (int w = 0; w < 32; ++w) t += ws[w][lane];
    g.out[(i / g.width) * g.out_stride + i % g.width] = t;
  }
}

}  // namespace

int proj_partials() { return kProjBlocks; }

template <int HM>
cudaError_t launch_ln_fwd_h(const ProjArgs &a, cudaStream_t stream) {
  const int blocks = kProjBlocks;
  if (a.cz % 64) return cudaErrorInvalidValue;
  switch (a.cz / 32) {
    case 2: ln_fwd_kernel<2, HM><<<blocks, 256, 0, stream>>>(a); break;
    case 4: ln_fwd_kernel<4, HM><<<blocks, 256, 0, stream>>>(a); break;
    case 6: ln_fwd_kernel<6, HM><<<blocks, 256, 0, stream>>>(a); break;
    case 8: ln_fwd_kernel<8, HM><<<blocks, 256, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_ln_fwd(const ProjArgs &a, cudaStream_t stream) {
  if (a.H < 1 || a.H > kMaxHeads) return cudaErrorInvalidValue;
  // one head (the multiplicative update's LayerNorms) skips three heads' dot products
  if (a.H == 1) return launch_ln_fwd_h<1>(a, stream);
  return a.H <= 4 ? launch_ln_fwd_h<4>(a, stream) : launch_ln_fwd_h<kMaxHeads>(a, stream);
}

template <int CPL, int HM>
cudaError_t launch_ln_bwd_k(const ProjArgs &a, cudaStream_t stream) {
  const uint32_t bytes = bwd_smem_bytes(a.cz);
  cudaError_t e = cudaFuncSetAttribute(ln_bwd_kernel<CPL, HM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  ln_bwd_kernel<CPL, HM><<<kProjBlocks, 256, bytes, stream>>>(a);
  return cudaGetLastError();
}

template <int HM>
cudaError_t launch_ln_bwd_h(const ProjArgs &a, cudaStream_t stream) {
  if (a.cz % 64) return cudaErrorInvalidValue;
  switch (a.cz / 32) {
    case 2: return launch_ln_bwd_k<2, HM>(a, stream);
    case 4: return launch_ln_bwd_k<4, HM>(a, stream);
    case 6: return launch_ln_bwd_k<6, HM>(a, stream);
    case 8: return launch_ln_bwd_k<8, HM>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_ln_bwd(const ProjArgs &a, cudaStream_t stream) {
  if (a.H < 1 || a.H > kMaxHeads) return cudaErrorInvalidValue;
  if (a.H == 1) return launch_ln_bwd_h<1>(a, stream);
  return a.H <= 4 ? launch_ln_bwd_h<4>(a, stream) : launch_ln_bwd_h<kMaxHeads>(a, stream);
}

cudaError_t launch_colsum(const __nv_bfloat16 *m, int64_t rows, int cols, float *part,
                          cudaStream_t stream) {
  const int blocks = kProjBlocks;
  if (cols % 64) return cudaErrorInvalidValue;
  switch (cols / 32) {
    case 2: colsum_kernel<2><<<blocks, 256, 0, stream>>>(m, rows, cols, part); break;
    case 4: colsum_kernel<4><<<blocks, 256, 0, stream>>>(m, rows, cols, part); break;
    case 6: colsum_kernel<6><<<blocks, 256, 0, stream>>>(m, rows, cols, part); break;
    case 8: colsum_kernel<8><<<blocks, 256, 0, stream>>>(m, rows, cols, part); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_ordered_sums(const SumSeg *segs, int nseg, cudaStream_t stream) {
  if (nseg < 1 || nseg > kMaxSumSegs) return cudaErrorInvalidValue;
  SumSegs ss{};
  ss.nseg = nseg;
  int64_t blocks = 0;
  for (int s = 0; s < nseg; ++s) {
    ss.seg[s] = segs[s];
    ss.first_block[s] = blocks;
    blocks += (segs[s].len + 31) / 32;
  }
  if (blocks == 0) return cudaSuccess;
  if (blocks >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  ordered_sum_kernel<<<(unsigned)blocks, 1024, 0, stream>>>(ss);
  return cudaGetLastError();
}

cudaError_t launch_ordered_sum(const float *part, int64_t n, int64_t part_stride, int64_t len,
                               float *out, int64_t width, int64_t out_stride,
                               cudaStream_t stream) {
  const SumSeg seg{part, n, part_stride, len, out, width, out_stride};
  return launch_ordered_sums(&seg, 1, stream);
}

}  // namespace tri
