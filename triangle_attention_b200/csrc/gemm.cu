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
// Persistent: one CTA per SM walks the output tiles (n fastest, then m, then
// the batch), so the tiles in flight at any moment are neighbours that share
// operands in L2. Tensor memory holds two 128 x 256 fp32 accumulators (all 512
// columns): either two consecutive 128 x 256 tiles, so the epilogue of one tile
// overlaps the main loop of the next, or the two 128-row halves of one
// 256 x 256 tile (the shapes are described at Pipe below).
//   warp 0      TMA producer: 64-wide K slices of X and Y, a ring of stages
//               running across tiles
//   warp 1      tensor-memory allocator and MMA issuer (N = 256 products)
//   warps 2..9  epilogue, two per accumulator lane quarter: tensor memory ->
//               bf16 or fp32 (32-column loads, the next one in flight while the
//               current one is converted) -> a staging ring of 4 KB boxes per
//               warp -> TMA stores (bf16: 64-column boxes, each routed to one
//               of up to four output tensors by its column; fp32: 32-column
//               boxes)
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "gemm.cuh"

namespace tri {
namespace {

constexpr int kTM = 128, kTK = 64;                     // rows of one accumulator; K slice
constexpr int kTN = 256;                               // output tile (128 or 256) x kTN
constexpr int kMaxStages = 4;
constexpr int kEpiWarps = 8;                           // two per accumulator lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 2 * kTN;                // two 128 x 256 accumulators
constexpr uint32_t kYBytes = kTN * kTK * 2;            // Y slice
constexpr uint32_t kAtomBytes = 64 * kTK * 2;          // one 64-wide MN atom column: 8 KB
constexpr uint32_t kBoxBytes = 32 * 128;               // staged output box: 32 rows x 128 B

// Shapes of the pipeline.
//  HALVES = 1: 128 x 256 tiles, the two accumulators hold consecutive tiles, so
//    one tile's epilogue overlaps the next tile's main loop. Short K (the
//    projections) takes 3 operand stages and two staged boxes per epilogue warp
//    (the epilogue is the longer part of a tile); long K with few rows (the
//    weight gradients) takes 4 stages and one box.
//  HALVES = 2: 256 x 256 tiles for long K and many rows (the triangle
//    multiplication): the two accumulators are the two 128-row halves of one
//    tile, so a K slice of Y feeds twice the MMA work and the operand traffic
//    per FLOP falls by a quarter; the epilogue no longer overlaps the main loop.
template <int STAGES, int RING, int HALVES>
struct Pipe {
  static constexpr int kTileM = kTM * HALVES;
  static constexpr int kBufs = HALVES == 1 ? 2 : 1;     // accumulator sets in TMEM
  static constexpr uint32_t kXBytes = kTileM * kTK * 2;
  static constexpr uint32_t kStageBytes = kXBytes + kYBytes;
  static constexpr uint32_t kOffStaging = STAGES * kStageBytes;
  static constexpr uint32_t kOffCtl = kOffStaging + kEpiWarps * RING * kBoxBytes;
};

struct __align__(8) GemmSmem {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t teardown;
  uint32_t tmem_base;
  uint32_t abort_flag;
};
template <int STAGES, int RING, int HALVES>
constexpr uint32_t smem_bytes() {
  return Pipe<STAGES, RING, HALVES>::kOffCtl + sizeof(GemmSmem) + 1024;   // +1024: alignment
}
static_assert(smem_bytes<4, 1, 1>() <= 227 * 1024 && smem_bytes<3, 2, 1>() <= 227 * 1024 &&
              smem_bytes<3, 1, 2>() <= 227 * 1024,
              "shared memory budget");

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

// Tile t of the walk: n fastest, then m, then the batch index.
struct Tile {
  int m0, n0, c;
};
__device__ __forceinline__ Tile tile_of(int t, int mt, int nt, int tile_m) {
  return {((t / nt) % mt) * tile_m, (t % nt) * kTN, t / (nt * mt)};
}

// K range of batch index c: split-K takes K columns [kbeg, kend) of operands
// that have no batch dimension of their own (their batch coordinate is 0);
// otherwise c is every tensor's batch coordinate.
struct KRange {
  int kbeg, nk, cin;
};
__device__ __forceinline__ KRange k_range(const GemmArgs &a, int c) {
  const int kbeg = a.k_split ? c * a.k_split : 0;
  const int kend = a.k_split ? min(a.K, kbeg + a.k_split) : a.K;
  return {kbeg, (kend - kbeg + kTK - 1) / kTK, a.k_split ? 0 : c};
}

// One 32-column chunk of a warp's 32 accumulator rows -> its staging box; a
// finished box goes out by TMA. bf16: two chunks fill a 64-column box; fp32:
// one chunk is a box. Every box commits one bulk group (empty when the box
// lies past the last output), so the ring's bulk_wait_read count is exact.
template <bool F32, int RING>
__device__ __forceinline__ void epilogue_chunk(const uint32_t (&v)[32], int cb, const Tile &tl,
                                               int row0, int lane, uint8_t *ring, uint32_t &nbox,
                                               const GemmOuts &outs, const GemmArgs &a) {
  const bool first_half = F32 || (cb & 1) == 0;
  uint8_t *box = ring + (nbox % RING) * kBoxBytes;
  if (first_half && nbox >= (uint32_t)RING) {
    if (lane == 0) bulk_wait_read<RING - 1>();       // the store from this slot has read it
    __syncwarp();
  }
  if (F32) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      *reinterpret_cast<uint4 *>(box + lane * 128 + ((q ^ (lane & 7)) << 4)) =
          make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else {
    float f[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
    const int col0 = tl.n0 + cb * 32;
    if (a.col_bias && col0 + 32 > a.col_bias_from) {
      if (col0 >= a.col_bias_from && col0 + 32 <= a.Nn) {
        // the whole chunk takes the bias: the same 32 floats for every lane
        const float4 *pb = reinterpret_cast<const float4 *>(a.col_bias + (col0 - a.col_bias_from));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 b = __ldg(pb + q);
          f[4 * q] += b.x, f[4 * q + 1] += b.y, f[4 * q + 2] += b.z, f[4 * q + 3] += b.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = col0 + e;
          if (col >= a.col_bias_from && col < a.Nn) f[e] += a.col_bias[col - a.col_bias_from];
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int chunk = (cb & 1) * 4 + q;             // 16-byte chunk of the 128-byte row
      *reinterpret_cast<uint4 *>(box + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
          make_uint4(pack_bf16(f[8 * q], f[8 * q + 1]), pack_bf16(f[8 * q + 2], f[8 * q + 3]),
                     pack_bf16(f[8 * q + 4], f[8 * q + 5]), pack_bf16(f[8 * q + 6], f[8 * q + 7]));
    }
  }
  if (F32 || (cb & 1)) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (F32) {
        tma_store_3d(&outs.map[0], box, tl.n0 + cb * 32, row0, tl.c);
      } else {
        const int n = tl.n0 + (cb >> 1) * 64;          // first column of the box
        const int o = n / a.cols_per_out;               // the output tensor it belongs to
        if (o < a.nouts) tma_store_3d(&outs.map[o], box, n - o * a.cols_per_out, row0, tl.c);
      }
      bulk_commit_group();
    }
    ++nbox;
  }
}

template <bool XMN, bool YMN, bool F32, int STAGES, int RING, int HALVES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ GemmMaps xs, const __grid_constant__ GemmMaps ys,
               const __grid_constant__ GemmOuts outs, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  using P = Pipe<STAGES, RING, HALVES>;
  GemmSmem &ctl = *reinterpret_cast<GemmSmem *>(smem + P::kOffCtl);
  volatile uint32_t *abort_flag = &ctl.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (a.M + P::kTileM - 1) / P::kTileM, nt = (a.Nn + kTN - 1) / kTN;
  const int tiles = mt * nt * a.batch;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    for (int b = 0; b < P::kBufs; ++b) {
      mbar_init(&ctl.acc_full[b], 1);
      mbar_init(&ctl.acc_empty[b], kEpiWarps);       // one arrival per epilogue warp
    }
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
      uint32_t it = 0;                                // K slices issued, over all tiles
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const Tile tl = tile_of(t, mt, nt, P::kTileM);
        const KRange kr = k_range(a, tl.c);
        for (int kt = 0; kt < kr.nk; ++kt, ++it) {
          const int st = it % STAGES;
          if (it >= (uint32_t)STAGES &&
              !wait_bar(&ctl.empty[st], ((it / STAGES) - 1) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          uint8_t *dst = smem + st * P::kStageBytes;
          mbar_arrive_expect_tx(&ctl.full[st], P::kStageBytes);
          const int k = kr.kbeg + kt * kTK;
          const int xi = k / a.k_per_x;                // the X tensor holding this K slice
          load_slice<XMN, P::kTileM>(dst, &xs.map[xi], &ctl.full[st], tl.m0,
                                     k - xi * a.k_per_x, kr.cin);
          if (a.n_per_y)
            load_y_slice<YMN>(dst + P::kXBytes, ys, a, &ctl.full[st], tl.n0, k, kr.cin);
          else
            load_slice<YMN, kTN>(dst + P::kXBytes, &ys.map[0], &ctl.full[st], tl.n0, k, kr.cin);
        }
      }
      if (!ok)      // let the copies already issued land before the CTA exits
        for (uint32_t j = (it > (uint32_t)STAGES ? it - STAGES : 0u); j < it; ++j)
          mbar_wait(&ctl.full[j % STAGES], (j / STAGES) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (elect_one()) {
      const uint32_t idesc = make_idesc_bf16(kTM, kTN, XMN, YMN);
      uint32_t it = 0;
      bool ok = true;
      int j = 0;                                      // tiles of this CTA
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
        const int buf = j % P::kBufs;
        const int use = j / P::kBufs;                 // earlier uses of this accumulator set
        if (use >= 1 &&
            !wait_bar(&ctl.acc_empty[buf], (use - 1) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const KRange kr = k_range(a, tile_of(t, mt, nt, P::kTileM).c);
        for (int kt = 0; kt < kr.nk; ++kt, ++it) {
          const int st = it % STAGES;
          if (!wait_bar(&ctl.full[st], (it / STAGES) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xa = smem_u32(smem + st * P::kStageBytes);
          const uint32_t ya = xa + P::kXBytes;
#pragma unroll
          for (int h = 0; h < HALVES; ++h) {
            // rows 128h.. of the X slice: 16 KB on in both layouts (K-major: the
            // second 128-row box; MN-major: the third 64-wide atom column)
            const uint32_t d = tmem + (buf * HALVES + h) * kTN;
#pragma unroll
            for (int ks = 0; ks < kTK / 16; ++ks)
              mma_ss(d, slice_desc<XMN>(xa + h * kTM * kTK * 2, ks), slice_desc<YMN>(ya, ks),
                     idesc, (kt > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&ctl.empty[st]);
        }
        if (ok) mma_commit(&ctl.acc_full[buf]);
      }
      // No tensor-memory operation may be in flight when the CTA tears down.
      mma_commit(&ctl.teardown);
      mbar_wait(&ctl.teardown, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    // Warp w reads accumulator lanes 32 (w % 4) .. + 31 (its rank in the
    // warpgroup). HALVES = 1: the first four epilogue warps take columns 0..127
    // of the tile, the other four columns 128..255. HALVES = 2: the first four
    // take the upper 128-row half, the other four the lower half, all columns.
    // Chunks past the output's last column (rounded up to a whole box) are
    // skipped.
    const int e = warp - 2, q4 = warp & 3, grp = e >> 2;
    uint8_t *ring = smem + P::kOffStaging + e * RING * kBoxBytes;
    uint32_t nbox = 0;
    int j = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
      const int buf = j % P::kBufs, par = (j / P::kBufs) & 1;
      bool ok = mbar_try_wait(&ctl.acc_full[buf], par) ||
                wait_bar(&ctl.acc_full[buf], par, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const Tile tl = tile_of(t, mt, nt, P::kTileM);
      const int acc = HALVES == 1 ? buf : grp;          // accumulator this warp drains
      const uint32_t ta = tmem + ((uint32_t)(q4 * 32) << 16) + acc * kTN;
      const int row0 = tl.m0 + (HALVES == 1 ? 0 : grp * kTM) + q4 * 32;
      const int cols = a.Nn - tl.n0;                   // output columns in this tile
      const int live = F32 ? (cols + 31) / 32 : 2 * ((cols + 63) / 64);
      const int cb0 = HALVES == 1 ? grp * (kTN / 64) : 0;
      const int cb1 = min(cb0 + (HALVES == 1 ? kTN / 64 : kTN / 32), live);
      if (cb0 < cb1 && row0 < a.M) {
        uint32_t va[32], vb[32];
        tmem_ld32_issue(ta + cb0 * 32, va);
        tmem_wait_ld32(va);
#pragma unroll 1
        for (int cb = cb0; cb < cb1; cb += 2) {
          const bool has_b = cb + 1 < cb1, has_a = cb + 2 < cb1;
          if (has_b) tmem_ld32_issue(ta + (cb + 1) * 32, vb);
          epilogue_chunk<F32, RING>(va, cb, tl, row0, lane, ring, nbox, outs, a);
          if (has_b) tmem_wait_ld32(vb);
          if (has_a) tmem_ld32_issue(ta + (cb + 2) * 32, va);
          if (has_b) epilogue_chunk<F32, RING>(vb, cb + 1, tl, row0, lane, ring, nbox, outs, a);
          if (has_a) tmem_wait_ld32(va);
        }
      }
      // every load of this accumulator is done: hand it back to the MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.acc_empty[buf]);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool XMN, bool YMN, bool F32, int STAGES, int RING, int HALVES>
cudaError_t launch_pipe(const GemmMaps &x, const GemmMaps &y, const GemmOuts &d,
                        const GemmArgs &args, int sms, cudaStream_t stream) {
  constexpr uint32_t bytes = smem_bytes<STAGES, RING, HALVES>();
  static_assert(bytes <= 227 * 1024, "shared memory budget");
  constexpr int tile_m = Pipe<STAGES, RING, HALVES>::kTileM;
  const int64_t tiles = (int64_t)((args.M + tile_m - 1) / tile_m) * ((args.Nn + kTN - 1) / kTN) *
                        args.batch;
  if (tiles >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  const int grid = (int)(tiles < sms ? tiles : sms);
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<XMN, YMN, F32, STAGES, RING, HALVES>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  gemm_tc_kernel<XMN, YMN, F32, STAGES, RING, HALVES><<<grid, kThreads, bytes, stream>>>(
      x, y, d, args);
  return cudaGetLastError();
}

template <bool XMN, bool YMN, bool F32>
cudaError_t launch(const GemmMaps &x, const GemmMaps &y, const GemmOuts &d,
                   const GemmArgs &args, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int k_tile = args.k_split ? args.k_split : args.K;   // K of one tile
  if ((k_tile + kTK - 1) / kTK < 8) return launch_pipe<XMN, YMN, F32, 3, 2, 1>(x, y, d, args, sms, stream);
  if (args.M <= kTM) return launch_pipe<XMN, YMN, F32, 4, 1, 1>(x, y, d, args, sms, stream);
  return launch_pipe<XMN, YMN, F32, 3, 1, 2>(x, y, d, args, sms, stream);
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
