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
//   dbias[h, xb, yb] += dS                         (tensor memory, all rows)
//
// The pair-bias gradient block stays in tensor memory for the whole row walk
// and is written once, so its sum over the rows runs in one fixed order. The
// dq contribution of the block still has to be summed with those of the other
// key tiles, the dk/dv contributions with those of the other query tiles: the
// block writes them (bf16) to per-tile partial tensors and a second kernel sums
// them in tile order. There are no floating-point atomics, so repeated calls
// are bit-identical.
//
// Warp roles (448 threads):
//   warp 0       TMA producer: Q, dU, K, V tiles, lse, D and mask bits of each
//                row; the bias block once
//   warp 1       tensor-memory allocator and MMA issuer
//   warps 2..5   elementwise, keys 0..63 of the block  (thread = query row)
//   warps 6..9   elementwise, keys 64..127
//   warps 10..13 partial writers (thread = tensor-memory lane of dQ/dK/dV)
//
// Tensor memory columns: S 0..127, dP 128..255, dbias 256..383,
// dQ 384..415, dK 416..447, dV 448..479.
#include <cmath>
#include <cstdint>
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
constexpr int kThreads = 448;
constexpr int kWriterWarp0 = 10;   // warps 10..13 write the tile partials
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDB = 256, kColDQ = 384, kColDK = 416,
                   kColDV = 448;
constexpr uint32_t kPairTileBytes = kBM * kC * 2;       // 8 KB
constexpr uint32_t kSqTileBytes = kBM * kBN * 2;        // 32 KB
// one pipeline stage: Q, dU, K, V tiles, then lse[128], D[128], 4 mask words
constexpr uint32_t kStLse = 4 * kPairTileBytes;
constexpr uint32_t kStD = kStLse + 512;
constexpr uint32_t kStMask = kStD + 512;
constexpr uint32_t kStageBytes = 34 * 1024;
constexpr uint32_t kOffIn = 0;
constexpr uint32_t kOffP = kOffIn + kStages * kStageBytes;
constexpr uint32_t kOffDS = kOffP + kSqTileBytes;
constexpr uint32_t kOffB = kOffDS + kSqTileBytes;
constexpr uint32_t kOffCtl = kOffB + kSqTileBytes;
constexpr float kLog2e = 1.4426950408889634f;

static_assert(kStMask + 16 <= kStageBytes, "stage overflow");
static_assert(kOffP % 1024 == 0 && kOffB % 1024 == 0, "swizzled tiles need 1 KB alignment");

struct __align__(8) BwdSmem {
  uint64_t in_full[kStages];
  uint64_t in_empty[kStages];
  uint64_t bias_full;
  uint64_t sdp_full, sdp_free;
  uint64_t pds_full, pds_free;
  uint64_t part_full, part_free;
  uint64_t final_bar, teardown;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

constexpr uint32_t kSmemBytes = kOffCtl + sizeof(BwdSmem) + 1024;

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

// Store 8 bf16 pairs of one row chunk into a 128x128 tile laid out as two
// 128-row x 128-byte halves with the 128-byte swizzle (chunk ^= row & 7).
__device__ __forceinline__ void st_tile_chunk(uint8_t *tile, int row, int half, int chunk,
                                              uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  uint8_t *p = tile + half * (kSqTileBytes / 2) + row * 128 + ((chunk ^ (row & 7)) << 4);
  *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}

// Probabilities and dS for NC keys of one row. MASKED selects the key-mask
// path (tail tiles, masked keys); the common path has none.
template <int NC, bool MASKED>
__device__ __forceinline__ void dsoftmax_chunk(const uint32_t (&s)[NC], const uint32_t (&dp)[NC],
                                               uint32_t (&db)[NC], const uint32_t (&bw)[NC / 2],
                                               uint32_t mbits, uint64_t c1x2, uint64_t nlx2,
                                               uint64_t ndx2, uint32_t (&pw)[NC / 2],
                                               uint32_t (&dw)[NC / 2]) {
  const uint64_t l2e2 = f2pack(kLog2e, kLog2e);
#pragma unroll
  for (int e = 0; e < NC; e += 2) {
    const uint64_t b2 = f2pack(bf16lo(bw[e / 2]), bf16hi(bw[e / 2]));
    const uint64_t bl2 = fma2(b2, l2e2, nlx2);
    const uint64_t t2 = fma2(f2pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c1x2, bl2);
    const float2 t = f2unpack(t2);
    float p0 = ex2_approx(t.x), p1 = ex2_approx(t.y);
    if (MASKED) {
      if (!((mbits >> e) & 1u)) p0 = 0.0f;
      if (!((mbits >> (e + 1)) & 1u)) p1 = 0.0f;
    }
    const uint64_t p2 = f2pack(p0, p1);
    const uint64_t d2 =
        mul2(p2, add2(f2pack(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])), ndx2));
    const float2 dsv = f2unpack(d2);
    const float2 dbv = f2unpack(add2(f2pack(__uint_as_float(db[e]), __uint_as_float(db[e + 1])), d2));
    db[e] = __float_as_uint(dbv.x);
    db[e + 1] = __float_as_uint(dbv.y);
    pw[e / 2] = pack_bf16_int(p0, p1);
    dw[e / 2] = pack_bf16_int(dsv.x, dsv.y);
  }
}

// 32 fp32 values (bit patterns) rounded to bf16, streamed to dst (64 bytes).
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16 *dst, const uint32_t (&v)[32]) {
  uint4 *op = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    __stcs(op + q, make_uint4(pack_bf16(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                              pack_bf16(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                              pack_bf16(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                              pack_bf16(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]))));
}

__global__ void __launch_bounds__(kThreads, 1)
bwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_du,
                const __grid_constant__ CUtensorMap tm_b, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  BwdSmem &ctl = *reinterpret_cast<BwdSmem *>(smem + kOffCtl);
  volatile uint32_t *abort_flag = &ctl.abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = a.N, H = a.H, nb = a.nb;
  const int xb = blockIdx.x, yb = blockIdx.y;
  const int h = blockIdx.z % H, g = blockIdx.z / H;
  const int r0 = g * a.rows_per_group;
  const int r1 = min(N, r0 + a.rows_per_group);
  const int T = max(0, r1 - r0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.in_full[s], 1);
      mbar_init(&ctl.in_empty[s], 1);
    }
    mbar_init(&ctl.bias_full, 1);
    mbar_init(&ctl.sdp_full, 1);
    mbar_init(&ctl.sdp_free, 256);
    mbar_init(&ctl.pds_full, 256);
    mbar_init(&ctl.pds_free, 1);
    mbar_init(&ctl.part_full, 1);
    mbar_init(&ctl.part_free, 128);
    mbar_init(&ctl.final_bar, 1);
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
      tma_load_3d(smem + kOffB, &tm_b, &ctl.bias_full, yb * kBN, xb * kBM, h);
      tma_load_3d(smem + kOffB + kSqTileBytes / 2, &tm_b, &ctl.bias_full, yb * kBN + 64, xb * kBM,
                  h);
      // lse and D rows of this query tile: min(128, N - x0) floats (N % 8 == 0)
      const uint32_t row_bytes = (uint32_t)min(kBM, N - xb * kBM) * 4u;
      for (int it = 0; it < T; ++it) {
        const int st = it % kStages;
        if (it >= kStages &&
            !wait_bar(&ctl.in_empty[st], ((it / kStages) - 1) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        const int r = r0 + it;
        uint8_t *in = smem + kOffIn + st * kStageBytes;
        mbar_arrive_expect_tx(&ctl.in_full[st], 4 * kPairTileBytes + 2 * row_bytes + 16);
        if (a.x_inner) {
          tma_load_4d(in, &tm_q, &ctl.in_full[st], 0, h, xb * kBM, r);
          tma_load_4d(in + 2 * kPairTileBytes, &tm_k, &ctl.in_full[st], 0, h, yb * kBN, r);
          tma_load_4d(in + 3 * kPairTileBytes, &tm_v, &ctl.in_full[st], 0, h, yb * kBN, r);
        } else {
          tma_load_4d(in, &tm_q, &ctl.in_full[st], 0, h, r, xb * kBM);
          tma_load_4d(in + 2 * kPairTileBytes, &tm_k, &ctl.in_full[st], 0, h, r, yb * kBN);
          tma_load_4d(in + 3 * kPairTileBytes, &tm_v, &ctl.in_full[st], 0, h, r, yb * kBN);
        }
        tma_load_4d(in + kPairTileBytes, &tm_du, &ctl.in_full[st], 0, h, xb * kBM, r);
        const int64_t lo = ((int64_t)r * H + h) * N + xb * kBM;
        bulk_load(in + kStLse, a.lse + lo, row_bytes, &ctl.in_full[st]);
        bulk_load(in + kStD, a.D + lo, row_bytes, &ctl.in_full[st]);
        bulk_load(in + kStMask, a.mask_bits + (int64_t)r * a.mask_bits_stride + yb * 4, 16,
                  &ctl.in_full[st]);
        armed[st] = it / kStages;
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
      auto issue_sdp = [&](int t) -> bool {
        const int st = t % kStages;
        if (!wait_bar(&ctl.in_full[st], (t / kStages) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t in = smem_u32(smem + kOffIn + st * kStageBytes);
        const uint32_t qa = in, ua = in + kPairTileBytes, ka = in + 2 * kPairTileBytes,
                       va = in + 3 * kPairTileBytes;
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_ss(tmem + kColS, make_sdesc(qa + ks * 32, 16, 512, kSwizzle64B),
                 make_sdesc(ka + ks * 32, 16, 512, kSwizzle64B), id_sp, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_ss(tmem + kColDP, make_sdesc(ua + ks * 32, 16, 512, kSwizzle64B),
                 make_sdesc(va + ks * 32, 16, 512, kSwizzle64B), id_sp, ks > 0 ? 1u : 0u);
        mma_commit(&ctl.sdp_full);
        return true;
      };
      auto issue_grads = [&](int t) -> bool {
        const int st = t % kStages;
        if (!wait_bar(&ctl.pds_full, t & 1, abort_flag, a.status)) return false;
        if (t >= 1 && !wait_bar(&ctl.part_free, (t - 1) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t in = smem_u32(smem + kOffIn + st * kStageBytes);
        const uint32_t qa = in, ua = in + kPairTileBytes, ka = in + 2 * kPairTileBytes;
        const uint32_t pa = smem_u32(smem + kOffP), da = smem_u32(smem + kOffDS);
        // dV = P^T dU and dK = dS^T Q: A is the [x][y] tile read MN-major (M = y),
        // B the [x][c] tile read MN-major (K = x).
#pragma unroll
        for (int ks = 0; ks < kBM / 16; ++ks)
          mma_ss(tmem + kColDV, make_sdesc(pa + ks * 2048, kSqTileBytes / 2, 1024, kSwizzle128B),
                 make_sdesc(ua + ks * 1024, 512, 512, kSwizzle64B), id_kv, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < kBM / 16; ++ks)
          mma_ss(tmem + kColDK, make_sdesc(da + ks * 2048, kSqTileBytes / 2, 1024, kSwizzle128B),
                 make_sdesc(qa + ks * 1024, 512, 512, kSwizzle64B), id_kv, ks > 0 ? 1u : 0u);
        // dQ = dS K: A is the [x][y] tile read K-major (K = y), B the [y][c] tile
        // read MN-major (K = y).
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_ss(tmem + kColDQ,
                 make_sdesc(da + (ks >> 2) * (kSqTileBytes / 2) + (ks & 3) * 32, 16, 1024,
                            kSwizzle128B),
                 make_sdesc(ka + ks * 1024, 512, 512, kSwizzle64B), id_q, ks > 0 ? 1u : 0u);
        mma_commit(&ctl.part_full);
        mma_commit(&ctl.pds_free);
        mma_commit(&ctl.in_empty[st]);
        return true;
      };
      bool ok = true;
      for (int it = 0; ok && it < T; ++it) {
        if (it >= 1) ok = wait_bar(&ctl.sdp_free, (it - 1) & 1, abort_flag, a.status);
        if (ok) ok = issue_sdp(it);
        if (ok && it >= 1) ok = issue_grads(it - 1);
      }
      if (ok && T > 0) ok = issue_grads(T - 1);
      mma_commit(&ctl.final_bar);
      mma_commit(&ctl.teardown);
      mbar_wait(&ctl.teardown, 0);
    }
  } else if (warp < kWriterWarp0) {
    // ---------------------------------------------------------- elementwise --
    const int wg = (warp - 2) >> 2;           // 0: keys 0..63, 1: keys 64..127
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const int x = xb * kBM + row;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t kbase = wg * 64;
    const uint64_t c1x2 = f2pack(a.scale * kLog2e, a.scale * kLog2e);
    bool ok = wait_bar_warp(&ctl.bias_full, 0, abort_flag, a.status);
    {
      uint32_t z[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) z[e] = 0u;
      tmem_st32(tl + kColDB + kbase, z);
      tmem_st32(tl + kColDB + kbase + 32, z);
      tmem_st_wait();
    }
    const uint8_t *brow = smem + kOffB + wg * (kSqTileBytes / 2) + row * 128;
    uint8_t *ptile = smem + kOffP;
    uint8_t *dstile = smem + kOffDS;
    for (int it = 0; ok && it < T; ++it) {
      const int st = it % kStages;
      if (!wait_bar_warp(&ctl.in_full[st], (it / kStages) & 1, abort_flag, a.status)) {
        ok = false;
        break;
      }
      const uint8_t *in = smem + kOffIn + st * kStageBytes;
      const float L = x < N ? reinterpret_cast<const float *>(in + kStLse)[row] : -INFINITY;
      const float Dx = x < N ? reinterpret_cast<const float *>(in + kStD)[row] : 0.0f;
      const uint32_t *mw = reinterpret_cast<const uint32_t *>(in + kStMask);
      const uint32_t m0 = mw[wg * 2], m1 = mw[wg * 2 + 1];
      const bool live = L > -INFINITY;
      const bool full = live && (m0 & m1) == 0xffffffffu;
      const float lL = live ? L * kLog2e : 0.0f;
      const uint64_t nlx2 = f2pack(-lL, -lL);
      const uint64_t ndx2 = f2pack(-Dx, -Dx);
      if (!wait_bar_warp(&ctl.sdp_full, it & 1, abort_flag, a.status)) { ok = false; break; }
      if (it >= 1 && !wait_bar_warp(&ctl.pds_free, (it - 1) & 1, abort_flag, a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        // 16 keys: kbase + 16*ch .. +15, i.e. 16-byte chunks 2*ch and 2*ch+1 of the half tile
        const uint32_t col = kbase + ch * 16;
        uint32_t s[16], dp[16], db[16], pw[8], dw[8], bw[8];
        tmem_ld16x3(tl + kColS + col, tl + kColDP + col, tl + kColDB + col, s, dp, db);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint4 bv =
              *reinterpret_cast<const uint4 *>(brow + (((2 * ch + q) ^ (row & 7)) << 4));
          bw[q * 4 + 0] = bv.x; bw[q * 4 + 1] = bv.y; bw[q * 4 + 2] = bv.z; bw[q * 4 + 3] = bv.w;
        }
        const uint32_t mbits = live ? (((ch < 2) ? m0 : m1) >> ((ch & 1) * 16)) : 0u;
        if (full)
          dsoftmax_chunk<16, false>(s, dp, db, bw, mbits, c1x2, nlx2, ndx2, pw, dw);
        else
          dsoftmax_chunk<16, true>(s, dp, db, bw, mbits, c1x2, nlx2, ndx2, pw, dw);
        tmem_st16(tl + kColDB + col, db);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          st_tile_chunk(ptile, row, wg, 2 * ch + q, pw[q * 4], pw[q * 4 + 1], pw[q * 4 + 2],
                        pw[q * 4 + 3]);
          st_tile_chunk(dstile, row, wg, 2 * ch + q, dw[q * 4], dw[q * 4 + 1], dw[q * 4 + 2],
                        dw[q * 4 + 3]);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctl.sdp_free);
      fence_proxy_async_smem();
      mbar_arrive(&ctl.pds_full);
    }
    // the pair-bias gradient block: summed over every row of the group
    if (ok) {
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t db[32];
        tmem_ld32(tl + kColDB + kbase + ch * 32, db);
        if (x >= N) continue;
        const int64_t hb = (int64_t)h * N * N;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int y = yb * kBN + kbase + ch * 32 + e;
          if (y >= N) break;
          const float val = __uint_as_float(db[e]);
          if (a.ngroups == 1)
            a.dbias[hb + (int64_t)x * a.bX + (int64_t)y * a.bY] = __float2bfloat16_rn(val);
          else
            a.part_db[((int64_t)g * H + h) * N * N + (int64_t)x * N + y] = val;
        }
      }
    }
  } else {
    // ------------------------------------------------------ partial writers --
    // The block's dq/dk/dv contributions, rounded to bf16, go to per-tile
    // partial tensors (compact variant frame); a separate kernel sums them in
    // tile order. Nothing here waits on global memory.
    const int q4 = warp & 3;
    const int lrow = q4 * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const int x = xb * kBM + lrow;
    const int y = yb * kBN + lrow;
    const int64_t pair = (int64_t)N * N * H * kC;
    for (int it = 0; it < T; ++it) {
      if (!wait_bar_warp(&ctl.part_full, it & 1, abort_flag, a.status)) break;
      tc_fence_after();
      uint32_t dq[32], dk[32], dv[32];
      tmem_ld32(tl + kColDQ, dq);
      tmem_ld32(tl + kColDK, dk);
      tmem_ld32(tl + kColDV, dv);
      tc_fence_before();
      mbar_arrive(&ctl.part_free);
      const int r = r0 + it;
      if (x < N)
        store_bf16x32(a.part_q + yb * pair + (((int64_t)r * N + x) * H + h) * kC, dq);
      if (y < N) {
        const int64_t off = xb * pair + (((int64_t)r * N + y) * H + h) * kC;
        store_bf16x32(a.part_k + off, dk);
        store_bf16x32(a.part_v + off, dv);
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

void bwd_bf16_plan(int N, int H, int *nxb, int *ngroups) {
  const int nb = (N + kBM - 1) / kBM;
  *nxb = nb;
  const int64_t tiles = (int64_t)nb * nb * H;
  int64_t g = tiles > 0 ? 148 / tiles : 1;
  if (g < 1) g = 1;
  if (g > N) g = N > 0 ? N : 1;
  const int rows = (int)((N + g - 1) / g);
  *ngroups = rows > 0 ? (N + rows - 1) / rows : 1;
}

cudaError_t launch_bwd_bf16(const BwdMaps &maps, const BwdArgs &args, cudaStream_t stream) {
  if (args.N == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(bwd_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(args.nb, args.nb, args.H * args.ngroups);
  bwd_bf16_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps.q, maps.k, maps.v, maps.du,
                                                           maps.bias, args);
  return cudaGetLastError();
}

}  // namespace tri
