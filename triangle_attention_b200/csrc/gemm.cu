// Batched bf16 GEMM on the sm_100a tensor cores, D[b][m][n] = sum_k X[b](m, k)
// Y[b](n, k) with fp32 accumulation in tensor memory. Each operand is read
// straight from its stored matrix, either K-major (the stored rows are m or n,
// k contiguous) or MN-major (the stored rows are k, m or n contiguous):
// tcgen05 takes both, so no operand is ever transposed in memory.
//
// It carries the triangle multiplicative update (each of its six products is
// one batch of per-channel N x N GEMMs) and the projections around the
// attention (LayerNorm output times the projection weights, and their
// gradients, the weight gradients as split-K batches of fp32 partial sums).
//
// One CTA computes one 128x256 tile of one batch (fp32 in tensor memory):
//   warp 0      TMA producer: 64-wide K slices of X and Y (48 KB), 2-stage ring
//   warp 1      tensor-memory allocator and MMA issuer (N = 256 products)
//   warps 2..5  epilogue: tensor memory -> bf16 or fp32 -> the idle stage
//               buffers -> TMA stores (bf16: 64-column boxes, each routed to one
//               of up to four output tensors by its column; fp32: 32-column
//               boxes)
// 96 KB of shared memory and 256 tensor-memory columns, so two CTAs share an
// SM and one's epilogue overlaps the other's main loop.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "gemm.cuh"

namespace tri {
namespace {

constexpr int kTM = 128, kTK = 64;
constexpr int kTN = 256;                               // output tile 128 x kTN
constexpr int kStages = 2;
constexpr int kMinBlocks = 2;                          // CTAs per SM the budget is sized for
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = kTN;
constexpr uint32_t kXBytes = kTM * kTK * 2;            // 16 KB X slice
constexpr uint32_t kYBytes = kTN * kTK * 2;            // Y slice
constexpr uint32_t kStageBytes = kXBytes + kYBytes;
constexpr uint32_t kOffCtl = kStages * kStageBytes;
constexpr uint32_t kAtomBytes = 64 * kTK * 2;          // one 64-wide MN atom column: 8 KB
constexpr uint32_t kWarpStage = 16 * 1024;             // epilogue staging per warp
static_assert(32 * kTN * 2 <= kWarpStage, "a warp's bf16 rows must fit its staging");
static_assert(4 * kWarpStage <= kStages * kStageBytes, "staging reuses the operand stages");

struct __align__(8) MulSmem {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint64_t teardown;
  uint32_t tmem_base;
  uint32_t abort_flag;
};
constexpr uint32_t kSmemBytes = kOffCtl + sizeof(MulSmem) + 1024;   // +1024 for alignment

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity,
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

// A ROWS x 64 operand slice into shared memory. K-major: ROWS/128 boxes of
// 64 (k) x 128 rows of the stored matrix (rows m or n, k contiguous), stacked.
// MN-major: ROWS/64 boxes of 64 (m or n) x 64 (k) of the stored matrix (rows k,
// m or n contiguous), one 8 KB atom column each.
template <bool MN, int ROWS>
__device__ __forceinline__ void load_slice(uint8_t *dst, const CUtensorMap *map, uint64_t *bar,
                                           int mn0, int k0, int c) {
  if (MN) {
#pragma unroll
    for (int h = 0; h < ROWS / 64; ++h) tma_load_3d(dst + h * kAtomBytes, map, bar, mn0 + 64 * h, k0, c);
  } else {
#pragma unroll
    for (int h = 0; h < ROWS / 128; ++h)
      tma_load_3d(dst + h * (128 * kTK * 2), map, bar, k0, mn0 + 128 * h, c);
  }
}

// The Y slice when Y is several tensors along n: each box (64 rows MN-major,
// 128 K-major) comes from the tensor holding its first row; rows past the last
// tensor read past its extent, which the copy fills with zeros.
template <bool MN>
__device__ __forceinline__ void load_y_slice(uint8_t *dst, const GemmMaps &ys, const GemmArgs &a,
                                             uint64_t *bar, int n0, int k0, int c) {
  constexpr int kBox = MN ? 64 : 128;
#pragma unroll
  for (int h = 0; h < kTN / kBox; ++h) {
    const int n = n0 + kBox * h;
    const int yi = min(n / a.n_per_y, a.ny - 1);
    load_slice<MN, kBox>(dst + h * (kBox * kTK * 2), &ys.map[yi], bar, n - yi * a.n_per_y, k0, c);
  }
}

// Descriptor of the 16-wide K step ks of a slice (128-byte swizzle). K-major:
// rows of 128 bytes, 8-row groups 1 KB apart, the K step 32 bytes along a row.
// MN-major: 64-wide MN atom columns 8 KB apart, 8 k-rows per 1 KB group, the K
// step 16 rows (2 KB).
template <bool MN>
__device__ __forceinline__ uint64_t slice_desc(uint32_t base, int ks) {
  return MN ? make_sdesc(base + ks * 2048, kAtomBytes, 1024, kSwizzle128B)
            : make_sdesc(base + ks * 32, 16, 1024, kSwizzle128B);
}

template <bool XMN, bool YMN, bool F32>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
gemm_tc_kernel(const __grid_constant__ GemmMaps xs, const __grid_constant__ GemmMaps ys,
               const __grid_constant__ GemmOuts outs, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  MulSmem &ctl = *reinterpret_cast<MulSmem *>(smem + kOffCtl);
  volatile uint32_t *abort_flag = &ctl.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTM, n0 = blockIdx.y * kTN, c = blockIdx.z;
  // split-K: batch index c takes K columns [kbeg, kend) of operands that have no
  // batch dimension of their own; otherwise c is every tensor's batch coordinate
  const int kbeg = a.k_split ? c * a.k_split : 0;
  const int kend = a.k_split ? min(a.K, kbeg + a.k_split) : a.K;
  const int cin = a.k_split ? 0 : c;
  const int nk = (kend - kbeg + kTK - 1) / kTK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    mbar_init(&ctl.acc_full, 1);
    mbar_init(&ctl.teardown, 1);
    ctl.abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (elect_one()) {
      tma_prefetch_desc(&xs.map[0]);
      tma_prefetch_desc(&ys.map[0]);
      int armed[kStages];
      for (int s = 0; s < kStages; ++s) armed[s] = -1;
      bool ok = true;
      for (int kt = 0; kt < nk; ++kt) {
        const int st = kt % kStages;
        if (kt >= kStages &&
            !wait_bar(&ctl.empty[st], ((kt / kStages) - 1) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        uint8_t *dst = smem + st * kStageBytes;
        mbar_arrive_expect_tx(&ctl.full[st], kStageBytes);
        const int k = kbeg + kt * kTK;
        const int xi = k / a.k_per_x;                  // the X tensor holding this K slice
        load_slice<XMN, kTM>(dst, &xs.map[xi], &ctl.full[st], m0, k - xi * a.k_per_x, cin);
        if (a.n_per_y)
          load_y_slice<YMN>(dst + kXBytes, ys, a, &ctl.full[st], n0, k, cin);
        else
          load_slice<YMN, kTN>(dst + kXBytes, &ys.map[0], &ctl.full[st], n0, k, cin);
        armed[st] = kt / kStages;
      }
      if (!ok)
        for (int s = 0; s < kStages; ++s)
          if (armed[s] >= 0) mbar_wait(&ctl.full[s], armed[s] & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (elect_one()) {
      const uint32_t idesc = make_idesc_bf16(kTM, kTN, XMN, YMN);
      bool ok = true;
      for (int kt = 0; kt < nk && ok; ++kt) {
        const int st = kt % kStages;
        if (!wait_bar(&ctl.full[st], (kt / kStages) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t xa = smem_u32(smem + st * kStageBytes);
        const uint32_t ya = xa + kXBytes;
#pragma unroll
        for (int ks = 0; ks < kTK / 16; ++ks)
          mma_ss(tmem, slice_desc<XMN>(xa, ks), slice_desc<YMN>(ya, ks), idesc,
                 (kt > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&ctl.empty[st]);
      }
      mma_commit(&ctl.acc_full);
      // No tensor-memory operation may be in flight when the CTA tears down.
      mma_commit(&ctl.teardown);
      mbar_wait(&ctl.teardown, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int q4 = warp & 3;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    bool ok = true;
    if (!mbar_try_wait(&ctl.acc_full, 0)) ok = wait_bar(&ctl.acc_full, 0, abort_flag, a.status);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      // The operand stages are idle once the accumulator is complete: each warp
      // stages its 32 rows there (boxes of 32 rows x 128 bytes, 128-byte
      // swizzle) and stores them with TMA, which clips rows and columns past the
      // output's extent.
      // 16 KB per warp: the four 64-column bf16 boxes of its rows, or a ring of
      // four 32-column fp32 boxes whose slot is reused once its store has read it
      uint8_t *stage = smem + q4 * kWarpStage;
#pragma unroll 1
      for (int cb = 0; cb < kTN / 32; ++cb) {
        uint32_t v[32];
        tmem_ld32(tl + cb * 32, v);
        if (F32) {
          // 32 fp32 columns = one 128-byte row of a box
          uint8_t *box = stage + (cb & 3) * (32 * 128);
          if (cb >= 4) {
            if (lane == 0) bulk_wait_read<3>();
            __syncwarp();
          }
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4 *>(box + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&outs.map[0], box, n0 + cb * 32, m0 + q4 * 32, c);
            bulk_commit_group();
          }
        } else {
          uint8_t *box = stage + (cb >> 1) * (32 * 128);
          if (a.col_bias) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = n0 + cb * 32 + e;
              if (col >= a.col_bias_from && col < a.Nn)
                v[e] = __float_as_uint(__uint_as_float(v[e]) + a.col_bias[col - a.col_bias_from]);
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (cb & 1) * 4 + q;       // 16-byte chunk of the 128-byte row
            *reinterpret_cast<uint4 *>(box + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                           pack_bf16(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                           pack_bf16(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                           pack_bf16(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
          }
          if (cb & 1) {
            fence_proxy_async_smem();
            __syncwarp();
            const int n = n0 + (cb >> 1) * 64;        // first column of the box
            const int o = n / a.cols_per_out;          // the output tensor it belongs to
            if (lane == 0 && o < a.nouts) {
              tma_store_3d(&outs.map[o], box, n - o * a.cols_per_out, m0 + q4 * 32, c);
              bulk_commit_group();
            }
          }
        }
      }
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool XMN, bool YMN, bool F32>
cudaError_t launch(const GemmMaps &x, const GemmMaps &y, const GemmOuts &d,
                   const GemmArgs &args, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<XMN, YMN, F32>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((args.M + kTM - 1) / kTM, (args.Nn + kTN - 1) / kTN, args.batch);
  gemm_tc_kernel<XMN, YMN, F32><<<grid, kThreads, kSmemBytes, stream>>>(x, y, d, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_tc(bool x_mn, bool y_mn, bool f32_out, const GemmMaps &x,
                           const GemmMaps &y, const GemmOuts &d, const GemmArgs &args,
                           cudaStream_t stream) {
  if (args.M == 0 || args.Nn == 0 || args.batch == 0) return cudaSuccess;
  // an empty K range would leave the accumulator unwritten: callers zero such outputs
  if (args.K <= 0 || (args.k_split && (args.k_split % kTK || (int64_t)(args.batch - 1) * args.k_split >= args.K)))
    return cudaErrorInvalidValue;
  if (args.k_per_x <= 0 || args.k_per_x % kTK) return cudaErrorInvalidValue;
  if (args.n_per_y && (args.ny < 1 || args.ny > 4 || args.n_per_y % (y_mn ? 64 : 128)))
    return cudaErrorInvalidValue;
  if (f32_out) {
    if (!x_mn && !y_mn) return launch<false, false, true>(x, y, d, args, stream);
    if (!x_mn && y_mn) return launch<false, true, true>(x, y, d, args, stream);
    if (x_mn && y_mn) return launch<true, true, true>(x, y, d, args, stream);
  } else {
    if (!x_mn && !y_mn) return launch<false, false, false>(x, y, d, args, stream);
    if (!x_mn && y_mn) return launch<false, true, false>(x, y, d, args, stream);
    if (x_mn && y_mn) return launch<true, true, false>(x, y, d, args, stream);
  }
  return cudaErrorInvalidValue;       // X MN-major with Y K-major: no product needs it
}

}  // namespace tri
