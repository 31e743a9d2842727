// bf16 backward of gated triangle self-attention on sm_100a (tcgen05 + TMA).
//
// Work unit: one CTA owns one (query tile xb, key tile yb, head h) block of the
// probability matrix and walks a group of attention rows in a fixed order. For
// every row it recomputes that 128x128 block of probabilities once, from the
// saved log-sum-exp, and reuses it for all four gradients ("TurboPairFormer
// accelera fino a 1,73x l'addestramento di OpenFold3 nei test", section
// "Dove si impiega il tempo"):
//   S  = Q K^T,  dP = dU V^T                       (tcgen05, tensor memory)
//   P  = exp(S c^-1/2 + b - lse),  dS = P (dP - D) (two elementwise warpgroups)
//   dV_t = P^T dU,  dK_t = dS^T Q,  dQ_t = dS K    (tcgen05)
//   dbias[h, xb, yb] += dS                         (registers, all rows)
//
// The pair-bias gradient block lives in the elementwise threads' registers for
// the whole row walk and is written once, so its sum over the rows runs in one
// fixed order. The dq contribution of the block still has to be summed with
// those of the other key tiles, the dk/dv contributions with those of the
// other query tiles: the block writes them (bf16) to per-tile partial tensors
// and a second kernel sums them in tile order. There are no floating-point
// atomics, so repeated calls are bit-identical.
//
// Pipeline: two S/dP buffers in tensor memory and two P/dS buffers in shared
// memory, so the tensor cores compute S/dP of the next row and the gradients of
// the previous row while the elementwise warps work on the current one. The
// gradient MMAs of row t write into the S columns of row t's buffer (already
// consumed); the elementwise warps move them out half-way through row t+1,
// which frees the buffer for row t+2.
//
// Warp roles (64 + 128 * kEltGroups threads):
//   warp 0      TMA producer: Q, dU, K, V tiles, lse, D and mask bits of each
//               row; the bias block once
//   warp 1      tensor-memory allocator and MMA issuer
//   warps 2..   kEltGroups elementwise warpgroups; warpgroup w handles the keys
//               kKeys*w .. kKeys*w + kKeys - 1 of the block (thread = query row)
//
// Tensor memory: buffer b (b = row & 1) at columns 256*b: S at +0..127, dP at
// +128..255; after the row's gradient MMAs, dQ at +0, dK at +32, dV at +64.
#include <cmath>
#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>

#include "bf16.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace tri {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kC = 32;
constexpr int kStages = 2;
constexpr int kEltGroups = 4;                            // elementwise warpgroups
constexpr int kKeys = 128 / kEltGroups;                  // keys of the block per group
constexpr int kThreads = 64 + kEltGroups * 128;
constexpr int kEltThreads = kEltGroups * 128;
// bf16 rounding of P and dS: on the integer pipes (true) or with cvt.rn (false)
constexpr bool kPackOnIntegerPipes = false;
// elementwise arithmetic on fp32 pairs (fma.rn.f32x2 and friends) or scalars
constexpr bool kPairArithmetic = true;
// chunk (of kKeys / 8) before which the elementwise warps drain the previous
// row's gradients: the last one. The gradient products of row t-1 start only
// when row t-1's P/dS are complete, so an earlier drain waits for them; a drain
// after the last chunk holds back the next S/dP products. Measured at N=768:
// last chunk 1.59 ms, staggered over chunks 2 and 3 1.74, after the row 1.70.
// (Read per warpgroup from a table: as a compile-time constant the drain is
// inlined into the unrolled chunk loop and the kernel spills.)
__device__ constexpr int kDrainChunk[4] = {3, 3, 3, 3};
static_assert(kEltGroups == 4 && kKeys / 8 == 4, "drain table written for four warpgroups");
// the producer asks L2 for the input tiles of row it + kL2Ahead while it loads
// row it (0: no prefetch)
constexpr int kL2Ahead = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBufCols = 256;
constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 0, kColDK = 32, kColDV = 64;
constexpr uint32_t kPairTileBytes = kBM * kC * 2;       // 8 KB
constexpr uint32_t kSqTileBytes = kBM * kBN * 2;        // 32 KB
// Shared memory (1 KB-aligned base, no slack: 231.6 KB of the 227 KiB limit):
//   P/dS buffer pb at kOffPD + pb*64K: P tile, then the dS tile (32 KB each)
//   the bias block (32 KB), read by the elementwise threads every row
//   input stage s: Q, dU, K, V tiles (32 KB) at kOffIn + s*32K
//   input stage s: lse[128], D[128], 4 mask words at kOffRow + s*kRowBytes
//   barriers
constexpr uint32_t kOffPD = 0;
constexpr uint32_t kPDBytes = 2 * kSqTileBytes;
constexpr uint32_t kOffBias = kOffPD + 2 * kPDBytes;
constexpr uint32_t kOffIn = kOffBias + kSqTileBytes;
constexpr uint32_t kStageBytes = 4 * kPairTileBytes;
constexpr uint32_t kRowBytes = 512 + 512 + 16;
constexpr uint32_t kOffRow = kOffIn + kStages * kStageBytes;
constexpr uint32_t kStLse = 0, kStD = 512, kStMask = 1024;   // within a row block
constexpr uint32_t kOffCtl = kOffRow + kStages * kRowBytes;
constexpr float kLog2e = 1.4426950408889634f;

static_assert(kOffBias % 1024 == 0 && kOffIn % 1024 == 0, "swizzled tiles need 1 KB alignment");
static_assert(kOffCtl % 8 == 0, "barriers need 8-byte alignment");

struct __align__(8) BwdSmem {
  uint64_t in_full[kStages];
  uint64_t in_empty[kStages];
  uint64_t bias_full;
  uint64_t sdp_full[2];      // S/dP of the row in TMEM buffer b are ready
  uint64_t pds_full[2];      // P/dS of the row in SMEM buffer pb are written
  uint64_t pds_free[2];      // gradient MMAs finished reading SMEM buffer pb
  uint64_t part_full[2];     // gradient partials in TMEM buffer b are ready
  uint64_t part_free[2];     // TMEM buffer b may be overwritten
  uint64_t teardown;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

constexpr uint32_t kSmemBytes = kOffCtl + sizeof(BwdSmem);
static_assert(kSmemBytes <= 227u * 1024u, "over the per-block shared memory limit");

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

__device__ __forceinline__ bool wait_bar_warp(uint64_t *bar, uint32_t parity,
                                              volatile uint32_t *abort_flag, int32_t *status) {
  const bool ok = wait_bar(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// 16 bytes (8 bf16 of one row) into a 128x128 tile laid out as two 128-row x
// 128-byte halves with the 128-byte swizzle (chunk ^= row & 7).
__device__ __forceinline__ void st_tile_chunk(uint8_t *tile, int row, int half, int chunk,
                                              uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  uint8_t *p = tile + half * (kSqTileBytes / 2) + row * 128 + ((chunk ^ (row & 7)) << 4);
  *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}

// NW fp32 values (bit patterns) rounded to bf16, streamed to dst (2*NW bytes).
template <int NW>
__device__ __forceinline__ void store_bf16(__nv_bfloat16 *dst, const uint32_t (&v)[NW]) {
  uint4 *op = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int q = 0; q < NW / 8; ++q)
    __stcs(op + q, make_uint4(pack_bf16(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                              pack_bf16(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                              pack_bf16(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                              pack_bf16(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]))));
}

// P and dS of 8 keys of one row (S and dP bits in sv/dpv, bias pairs bw[0..3]),
// dbias pairs db2[0..3] += dS. MASKED: keys whose bit in mbits is clear get 0.
template <bool MASKED>
__device__ __forceinline__ void dsoftmax8(const uint32_t (&sv)[8], const uint32_t (&dpv)[8],
                                          const uint32_t *bw, uint64_t *db2, uint32_t mbits,
                                          uint64_t c1x2, uint64_t l2e2, uint64_t nlx2,
                                          uint64_t ndx2, uint32_t (&pw)[4], uint32_t (&dw)[4]) {
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const uint32_t b = bw[e / 2];
    float p0, p1;
    float2 ds;
    if (kPairArithmetic) {
      const uint64_t bl2 = fma2(f2pack(bf16lo(b), bf16hi(b)), l2e2, nlx2);
      const float2 t =
          f2unpack(fma2(f2pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c1x2, bl2));
      p0 = ex2_approx(t.x);
      p1 = ex2_approx(t.y);
      if (MASKED) {
        if (!((mbits >> e) & 1u)) p0 = 0.0f;
        if (!((mbits >> (e + 1)) & 1u)) p1 = 0.0f;
      }
      const uint64_t ds2 =
          mul2(f2pack(p0, p1),
               add2(f2pack(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])), ndx2));
      db2[e / 2] = add2(db2[e / 2], ds2);
      ds = f2unpack(ds2);
    } else {
      const float c1 = f2unpack(c1x2).x, nl = f2unpack(nlx2).x, nd = f2unpack(ndx2).x;
      p0 = ex2_approx(fmaf(__uint_as_float(sv[e]), c1, fmaf(bf16lo(b), kLog2e, nl)));
      p1 = ex2_approx(fmaf(__uint_as_float(sv[e + 1]), c1, fmaf(bf16hi(b), kLog2e, nl)));
      if (MASKED) {
        if (!((mbits >> e) & 1u)) p0 = 0.0f;
        if (!((mbits >> (e + 1)) & 1u)) p1 = 0.0f;
      }
      ds.x = p0 * (__uint_as_float(dpv[e]) + nd);
      ds.y = p1 * (__uint_as_float(dpv[e + 1]) + nd);
      const float2 acc = f2unpack(db2[e / 2]);
      db2[e / 2] = f2pack(acc.x + ds.x, acc.y + ds.y);
    }
    if (kPackOnIntegerPipes) {
      pw[e / 2] = pack_bf16_int(p0, p1);
      dw[e / 2] = pack_bf16_int(ds.x, ds.y);
    } else {
      pw[e / 2] = pack_bf16(p0, p1);
      dw[e / 2] = pack_bf16(ds.x, ds.y);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
bwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_du,
                const __grid_constant__ CUtensorMap tm_b, const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    // the layout has no room for realignment: refuse rather than misplace tiles
    if (threadIdx.x == 0) report_status(a.status, kStatusBounds);
    return;
  }
  BwdSmem &ctl = *reinterpret_cast<BwdSmem *>(smem + kOffCtl);
  volatile uint32_t *abort_flag = &ctl.abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = a.N, H = a.H;
  const int xb = blockIdx.x, yb = blockIdx.y;
  // blockIdx.z = (problem pb, row group g, head h), h fastest; rows count on
  // across the problems of a batch (row pb*N + r is row r of problem pb)
  const int h = blockIdx.z % H, g = (blockIdx.z / H) % a.ngroups, pb = blockIdx.z / H / a.ngroups;
  const int r0 = a.row0 + pb * N + g * a.rows_per_group;
  const int r1 = min(min(a.row_end, (pb + 1) * N), r0 + a.rows_per_group);
  const int T = max(0, r1 - r0);
  const int rb0 = r0 - pb * N;        // r0's row inside its problem

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.in_full[s], 1);
      mbar_init(&ctl.in_empty[s], 1);
    }
    mbar_init(&ctl.bias_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl.sdp_full[b], 1);
      mbar_init(&ctl.pds_full[b], kEltThreads);
      mbar_init(&ctl.pds_free[b], 1);
      mbar_init(&ctl.part_full[b], 1);
      mbar_init(&ctl.part_free[b], kEltThreads);
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
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_du);
      tma_prefetch_desc(&tm_b);
      int armed[kStages];
      for (int s = 0; s < kStages; ++s) armed[s] = -1;
      bool ok = true;
      mbar_arrive_expect_tx(&ctl.bias_full, kSqTileBytes);
      tma_load_3d(smem + kOffBias, &tm_b, &ctl.bias_full, yb * kBN, xb * kBM, pb * H + h);
      tma_load_3d(smem + kOffBias + kSqTileBytes / 2, &tm_b, &ctl.bias_full, yb * kBN + 64,
                  xb * kBM, pb * H + h);
      // lse and D rows of this query tile: min(128, N - x0) floats (N % 8 == 0)
      const uint32_t row_bytes = (uint32_t)min(kBM, N - xb * kBM) * 4u;
      for (int it = 0; it < T; ++it) {
        const int st = it % kStages;
        if (it >= kStages &&
            !wait_bar(&ctl.in_empty[st], ((it / kStages) - 1) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        const int r = r0 + it, rb = rb0 + it;
        uint8_t *in = smem + kOffIn + st * kStageBytes;
        mbar_arrive_expect_tx(&ctl.in_full[st], 4 * kPairTileBytes + 2 * row_bytes + 16);
        if (a.x_inner) {
          tma_load_5d(in, &tm_q, &ctl.in_full[st], 0, h, xb * kBM, rb, pb);
          tma_load_5d(in + 2 * kPairTileBytes, &tm_k, &ctl.in_full[st], 0, h, yb * kBN, rb, pb);
          tma_load_5d(in + 3 * kPairTileBytes, &tm_v, &ctl.in_full[st], 0, h, yb * kBN, rb, pb);
        } else {
          tma_load_5d(in, &tm_q, &ctl.in_full[st], 0, h, rb, xb * kBM, pb);
          tma_load_5d(in + 2 * kPairTileBytes, &tm_k, &ctl.in_full[st], 0, h, rb, yb * kBN, pb);
          tma_load_5d(in + 3 * kPairTileBytes, &tm_v, &ctl.in_full[st], 0, h, rb, yb * kBN, pb);
        }
        tma_load_5d(in + kPairTileBytes, &tm_du, &ctl.in_full[st], 0, h, xb * kBM, rb, pb);
        const int64_t lo = ((int64_t)r * H + h) * N + xb * kBM;
        uint8_t *rd = smem + kOffRow + st * kRowBytes;
        bulk_load(rd + kStLse, a.lse + lo, row_bytes, &ctl.in_full[st]);
        bulk_load(rd + kStD, a.D + lo, row_bytes, &ctl.in_full[st]);
        bulk_load(rd + kStMask,
                  a.mask_bits + (int64_t)(a.mask_per_row ? r : pb) * a.mask_bits_stride + yb * 4,
                  16,
                  &ctl.in_full[st]);
        armed[st] = it / kStages;
        if (kL2Ahead > 0 && it + kL2Ahead < T) {
          const int rp = r + kL2Ahead, rbp = rb + kL2Ahead;
          if (a.x_inner) {
            tma_prefetch_l2_5d(&tm_q, 0, h, xb * kBM, rbp, pb);
            tma_prefetch_l2_5d(&tm_k, 0, h, yb * kBN, rbp, pb);
            tma_prefetch_l2_5d(&tm_v, 0, h, yb * kBN, rbp, pb);
          } else {
            tma_prefetch_l2_5d(&tm_q, 0, h, rbp, xb * kBM, pb);
            tma_prefetch_l2_5d(&tm_k, 0, h, rbp, yb * kBN, pb);
            tma_prefetch_l2_5d(&tm_v, 0, h, rbp, yb * kBN, pb);
          }
          tma_prefetch_l2_5d(&tm_du, 0, h, xb * kBM, rbp, pb);
          const int64_t lp = ((int64_t)rp * H + h) * N + xb * kBM;
          bulk_prefetch_l2(a.lse + lp, row_bytes);
          bulk_prefetch_l2(a.D + lp, row_bytes);
        }
      }
      if (!ok) {
        mbar_wait(&ctl.bias_full, 0);
        for (int s = 0; s < kStages; ++s)
          if (armed[s] >= 0) mbar_wait(&ctl.in_full[s], armed[s] & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (elect_one()) {
      const uint32_t id_sp = make_idesc_bf16(kBM, kBN, false, false);
      const uint32_t id_kv = make_idesc_bf16(kBN, kC, true, true);
      const uint32_t id_q = make_idesc_bf16(kBM, kC, false, true);
      // S and dP of row t into TMEM buffer t & 1
      auto issue_sdp = [&](int t) -> bool {
        const int st = t % kStages, b = t & 1;
        if (t >= 2 && !wait_bar(&ctl.part_free[b], ((t >> 1) - 1) & 1, abort_flag, a.status))
          return false;
        if (!wait_bar(&ctl.in_full[st], (t / kStages) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t in = smem_u32(smem + kOffIn + st * kStageBytes);
        const uint32_t qa = in, ua = in + kPairTileBytes, ka = in + 2 * kPairTileBytes,
                       va = in + 3 * kPairTileBytes;
        const uint32_t tb = tmem + b * kBufCols;
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_ss(tb + kColS, make_sdesc(qa + ks * 32, 16, 512, kSwizzle64B),
                 make_sdesc(ka + ks * 32, 16, 512, kSwizzle64B), id_sp, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_ss(tb + kColDP, make_sdesc(ua + ks * 32, 16, 512, kSwizzle64B),
                 make_sdesc(va + ks * 32, 16, 512, kSwizzle64B), id_sp, ks > 0 ? 1u : 0u);
        mma_commit(&ctl.sdp_full[b]);
        return true;
      };
      // dV, dK, dQ of row t from its P/dS (SMEM buffer t & 1) into the S
      // columns of TMEM buffer t & 1
      auto issue_grads = [&](int t) -> bool {
        const int st = t % kStages, b = t & 1;
        if (!wait_bar(&ctl.pds_full[b], (t >> 1) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t in = smem_u32(smem + kOffIn + st * kStageBytes);
        const uint32_t qa = in, ua = in + kPairTileBytes, ka = in + 2 * kPairTileBytes;
        const uint32_t pa = smem_u32(smem + kOffPD + b * kPDBytes);
        const uint32_t da = pa + kSqTileBytes;
        const uint32_t tb = tmem + b * kBufCols;
        // dV = P^T dU and dK = dS^T Q: A is the [x][y] tile read MN-major (M = y),
        // B the [x][c] tile read MN-major (K = x).
#pragma unroll
        for (int ks = 0; ks < kBM / 16; ++ks)
          mma_ss(tb + kColDV, make_sdesc(pa + ks * 2048, kSqTileBytes / 2, 1024, kSwizzle128B),
                 make_sdesc(ua + ks * 1024, 512, 512, kSwizzle64B), id_kv, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < kBM / 16; ++ks)
          mma_ss(tb + kColDK, make_sdesc(da + ks * 2048, kSqTileBytes / 2, 1024, kSwizzle128B),
                 make_sdesc(qa + ks * 1024, 512, 512, kSwizzle64B), id_kv, ks > 0 ? 1u : 0u);
        // dQ = dS K: A is the [x][y] tile read K-major (K = y), B the [y][c] tile
        // read MN-major (K = y).
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_ss(tb + kColDQ,
                 make_sdesc(da + (ks >> 2) * (kSqTileBytes / 2) + (ks & 3) * 32, 16, 1024,
                            kSwizzle128B),
                 make_sdesc(ka + ks * 1024, 512, 512, kSwizzle64B), id_q, ks > 0 ? 1u : 0u);
        mma_commit(&ctl.part_full[b]);
        mma_commit(&ctl.pds_free[b]);
        mma_commit(&ctl.in_empty[st]);
        return true;
      };
      bool ok = true;
      for (int it = 0; ok && it < T; ++it) {
        ok = issue_sdp(it);
        if (ok && it >= 1) ok = issue_grads(it - 1);
      }
      if (ok && T > 0) ok = issue_grads(T - 1);
      mma_commit(&ctl.teardown);
      mbar_wait(&ctl.teardown, 0);
    }
  } else {
    // ---------------------------------------------------------- elementwise --
    const int wg = (warp - 2) >> 2;           // keys kKeys*wg .. of the block
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;           // query row of the block = TMEM lane
    const int x = xb * kBM + row;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t kbase = wg * kKeys;
    const int half = kbase / 64, chunk0 = (kbase % 64) / 8;   // place in the P/dS tiles
    const uint64_t c1x2 = f2pack(a.scale * kLog2e, a.scale * kLog2e);
    const uint64_t l2e2 = f2pack(kLog2e, kLog2e);
    bool ok = wait_bar_warp(&ctl.bias_full, 0, abort_flag, a.status);
    // this thread's kKeys dbias sums (fp32 pairs); its bias row stays in shared memory
    uint64_t dbias2[kKeys / 2];
#pragma unroll
    for (int e = 0; e < kKeys / 2; ++e) dbias2[e] = 0ull;
    const uint8_t *brow = smem + kOffBias + half * (kSqTileBytes / 2) + row * 128;
    // 16-byte chunk chunk0 + ch of the swizzled row is at (cswz ^ ch) (chunk0 is a
    // multiple of kKeys / 8, so adding ch never carries into its bits)
    const uint32_t cswz = (uint32_t)(chunk0 ^ (row & 7));
    const int drain_chunk = kDrainChunk[wg];
    static_assert((kKeys / 8 & (kKeys / 8 - 1)) == 0, "key groups must be powers of two");

    // Gradient pieces: piece j (0..5) is the 16 channels 16*(j&1).. of dQ (j < 2),
    // dK (j < 4) or dV, for this warp's 32 lanes; warpgroup wg owns the pieces
    // j = wg, wg + kEltGroups, ... A piece of row r is one tile's contribution:
    // dQ of query tile xb (to be summed over key tiles), dK/dV of key tile yb (to
    // be summed over query tiles). Contributions are stored piece-major,
    // [t][r][h][j&1][i][16] (t the tile summed over, i the query or key): a lane
    // writes its 16 channels with one 32-byte store and a warp store covers 1 KB.
    const int64_t pair = (int64_t)a.B * N * N * H * kC;   // one tile's contributions
    // piece j's 16-channel plane of row r in one tensor's contributions
    auto piece_base = [&](int j, int r) -> __nv_bfloat16 * {
      __nv_bfloat16 *buf = j < 2 ? a.part_q : j < 4 ? a.part_k : a.part_v;
      return buf + ((((int64_t)r * H + h) * 2 + (j & 1)) * N) * 16;
    };

    // Row t's pieces from TMEM buffer t & 1 to this tile's contribution slots.
    auto drain = [&](int t) -> bool {
      const int b = t & 1;
      if (!wait_bar_warp(&ctl.part_full[b], (t >> 1) & 1, abort_flag, a.status)) return false;
      tc_fence_after();
      const uint32_t tb = tl + b * kBufCols;
      const int r = r0 + t;
      for (int j = wg; j < 6; j += kEltGroups) {
        const uint32_t col = j < 2 ? kColDQ + 16 * j : j < 4 ? kColDK + 16 * (j - 2)
                                                             : kColDV + 16 * (j - 4);
        const int i = (j < 2 ? xb : yb) * kBM + row;
        const int tsum = j < 2 ? yb : xb;
        uint32_t w[8];
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {     // 8 columns at a time keeps registers low
          uint32_t v[8];
          tmem_ld8(tb + col + 8 * c8, v);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[4 * c8 + e] = pack_bf16(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        }
        if (i < N) st_global_cs_v8(piece_base(j, r) + tsum * pair + (int64_t)i * 16, w);
      }
      tc_fence_before();
      mbar_arrive(&ctl.part_free[b]);
      return true;
    };

    for (int it = 0; ok && it < T; ++it) {
      const int st = it % kStages, b = it & 1;
      if (!wait_bar_warp(&ctl.in_full[st], (it / kStages) & 1, abort_flag, a.status)) {
        ok = false;
        break;
      }
      const uint8_t *in = smem + kOffRow + st * kRowBytes;
      const float L = x < N ? reinterpret_cast<const float *>(in + kStLse)[row] : -INFINITY;
      const float Dx = x < N ? reinterpret_cast<const float *>(in + kStD)[row] : 0.0f;
      // key bits of this warpgroup's keys: kKeys / 32 words from word kbase / 32
      const uint4 mw4 = *reinterpret_cast<const uint4 *>(in + kStMask);
      uint32_t kw[kKeys / 32];
      uint32_t mall = 0xffffffffu;
#pragma unroll
      for (int w = 0; w < kKeys / 32; ++w) {
        const int i = (int)(kbase / 32) + w;
        kw[w] = i == 0 ? mw4.x : i == 1 ? mw4.y : i == 2 ? mw4.z : mw4.w;
        mall &= kw[w];
      }
      const bool live = L > -INFINITY;
      // The unmasked form runs only when every lane of the warp may take it: the
      // per-row body holds warp-collective tensor-memory loads and waits, so the
      // choice must be warp-uniform (lanes past N in a ragged tile are not live).
      const bool full = __all_sync(0xffffffffu, live && mall == 0xffffffffu);
      const float lL = live ? L * kLog2e : 0.0f;
      const uint64_t nlx2 = f2pack(-lL, -lL);
      const uint64_t ndx2 = f2pack(-Dx, -Dx);
      if (!wait_bar_warp(&ctl.sdp_full[b], (it >> 1) & 1, abort_flag, a.status) ||
          (it >= 2 && !wait_bar_warp(&ctl.pds_free[b], ((it >> 1) - 1) & 1, abort_flag, a.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint8_t *ptile = smem + kOffPD + b * kPDBytes;
      uint8_t *dstile = ptile + kSqTileBytes;
      const uint32_t sb = tl + b * kBufCols + kColS + kbase;
      const uint32_t db = tl + b * kBufCols + kColDP + kbase;
      // One row's kKeys keys, 8 at a time; the S/dP loads of the next 8 are in
      // flight while these are processed. The masked form is chosen per row.
      auto row_keys = [&](auto masked_tag) -> bool {
        constexpr bool kMasked = decltype(masked_tag)::value;
        uint32_t sv[2][8], dpv[2][8];
        tmem_ld8x2_issue(sb, db, sv[0], dpv[0]);
        tmem_wait_ld8x2(sv[0], dpv[0]);
#pragma unroll
        for (int ch = 0; ch < kKeys / 8; ++ch) {
          const int cur = ch & 1, nxt = cur ^ 1;
          if (ch == drain_chunk && it >= 1) {
            // the previous row's gradients are done by now
            if (!drain(it - 1)) return false;
          }
          if (ch + 1 < kKeys / 8)
            tmem_ld8x2_issue(sb + (ch + 1) * 8, db + (ch + 1) * 8, sv[nxt], dpv[nxt]);
          const uint4 bv = *reinterpret_cast<const uint4 *>(brow + ((cswz ^ ch) << 4));
          const uint32_t bias[4] = {bv.x, bv.y, bv.z, bv.w};
          uint32_t mbits = 0u;
          if (kMasked) mbits = live ? (kw[(8 * ch) / 32] >> ((8 * ch) % 32)) : 0u;
          uint32_t pw[4], dw[4];
          dsoftmax8<kMasked>(sv[cur], dpv[cur], bias, dbias2 + ch * 4, mbits, c1x2, l2e2, nlx2,
                             ndx2, pw, dw);
          st_tile_chunk(ptile, row, half, chunk0 + ch, pw[0], pw[1], pw[2], pw[3]);
          st_tile_chunk(dstile, row, half, chunk0 + ch, dw[0], dw[1], dw[2], dw[3]);
          if (ch + 1 < kKeys / 8) tmem_wait_ld8x2(sv[nxt], dpv[nxt]);
        }
        return true;
      };
      ok = full ? row_keys(std::false_type{}) : row_keys(std::true_type{});
      if (!ok) break;
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&ctl.pds_full[b]);
    }
    if (ok && T > 0) ok = drain(T - 1);
    // the pair-bias gradient block: summed over every row of the group
    if (ok && x < N) {
      const int64_t hb = ((int64_t)pb * H + h) * N * N;
      const int y0 = yb * kBN + kbase;
#pragma unroll
      for (int e = 0; e < kKeys; e += 2) {
        const float2 v = f2unpack(dbias2[e / 2]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int y = y0 + e + u;
          const float val = u ? v.y : v.x;
          if (y < N) {
            if (a.dbias)
              a.dbias[hb + (int64_t)x * a.bX + (int64_t)y * a.bY] = __float2bfloat16_rn(val);
            else
              a.part_db[(((int64_t)g * a.B + pb) * H + h) * N * N + (int64_t)x * N + y] = val;
          }
        }
      }
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

}  // namespace

int bwd_bf16_max_groups(int N, int H) {
  const int nb = (N + kBM - 1) / kBM;
  const int64_t tiles = (int64_t)nb * nb * H;
  int64_t g = tiles > 0 ? 148 / tiles : 1;
  if (g < 1) g = 1;
  if (g > N) g = N > 0 ? N : 1;
  return (int)g;
}

void bwd_bf16_plan(int N, int H, int rows, int *nxb, int *ngroups) {
  const int nb = (N + kBM - 1) / kBM;
  *nxb = nb;
  int64_t g = bwd_bf16_max_groups(N, H);
  if (g > rows) g = rows > 0 ? rows : 1;
  const int per = (int)((rows + g - 1) / g);
  *ngroups = per > 0 ? (rows + per - 1) / per : 1;
}

cudaError_t launch_bwd_bf16(const BwdMaps &maps, const BwdArgs &args, cudaStream_t stream) {
  if (args.N == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(bwd_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(args.nb, args.nb, args.H * args.ngroups * args.B);
  bwd_bf16_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps.q, maps.k, maps.v, maps.du,
                                                           maps.bias, args);
  return cudaGetLastError();
}

}  // namespace tri
