// bf16 forward of gated triangle self-attention on sm_100a (tcgen05 + TMA).
//
// Work unit: one CTA owns (query tile of 128, head h, group of 8 attention
// rows). The N^3*H logits never leave the chip: for each key tile of 64 the CTA
// stages the 128x64 pair-bias tile once by TMA (shared by all 8 rows, since the
// bias does not depend on the row) and then, row by row, computes S = Q K^T on
// the tensor cores into tensor memory, turns it into probabilities with an
// online softmax, and accumulates O += P V in tensor memory. The probabilities
// never exist as a whole: each tile is produced and consumed on chip
// ("MegaFold: Efficient Training of Next-Generation 3D Attention Protein Models
// on Cross-Platform GPUs", tool 1, EvoFlash-3D). The sigmoid gate, the key mask
// and the log-sum-exp save are fused into the same kernel ("HelixFold: An
// Efficient Implementation of AlphaFold2 using PaddlePaddle", proposed methods:
// fused gated self-attention).
//
// Warp roles (576 threads):
//   warp 0       TMA producer (one elected lane)
//   warp 1       tensor-memory allocator and MMA issuer (one elected lane)
//   warps 2..17  four softmax / epilogue warpgroups; warpgroup w owns rows w and
//                w + 4 of the CTA and the S buffer w
// In a warpgroup, thread = query row of the tile (tensor-memory lane), so the
// row max and row sum are thread-local. The four warpgroups cycle through their
// rows independently: while one waits for the tensor cores (its P V product and
// its next S), the other three turn their S tiles into probabilities.
//
// Tensor memory (512 columns): S buffer w (64 fp32 columns) at 64*w; the bf16
// probabilities overwrite its first 32 columns and feed the PV product straight
// from tensor memory. O accumulators of the 8 rows at 256 + 32*rr.
#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "bf16.cuh"
#include "ptx.cuh"

namespace tri {
namespace {

constexpr int kBM = 128;          // queries per tile
constexpr int kBN = 64;           // keys per tile
constexpr int kC = 32;            // head dimension
constexpr int kRows = 8;          // attention rows per CTA
constexpr int kGroups = 4;        // softmax warpgroups; warpgroup w owns rows w, w + 4
constexpr int kStages = 8;        // K/V pipeline depth (each stage 8 KB)
constexpr int kThreads = 64 + 128 * kGroups;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = kGroups * kBN;           // 256
constexpr uint32_t kQTileBytes = kBM * kC * 2;      // 8 KB
constexpr uint32_t kKVTileBytes = kBN * kC * 2;     // 4 KB
constexpr uint32_t kBiasTileBytes = kBM * kBN * 2;  // 16 KB: 128 rows of 128 bytes
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// bf16 rounding of P: on the integer pipes (true) or with cvt.rn (false)
constexpr bool kPackOnIntegerPipes = false;
static_assert(kRows == 2 * kGroups, "each warpgroup owns two rows");

struct __align__(8) FwdSmem {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t bias_full[2];
  uint64_t bias_empty[2];
  uint64_t s_full[kGroups];
  uint64_t p_full[kGroups];
  uint64_t o_done[kRows];
  uint64_t o_final;
  uint64_t teardown;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kRows * kQTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kKVTileBytes;
constexpr uint32_t kOffB = kOffV + kStages * kKVTileBytes;
constexpr uint32_t kOffMask = kOffB + 2 * kBiasTileBytes;   // 16 bytes of key bits per stage
constexpr uint32_t kOffCtl = kOffMask + kStages * 16;
constexpr uint32_t kSmemBytes = kOffCtl + sizeof(FwdSmem) + 1024;  // +1024 for alignment
static_assert(kOffB % 1024 == 0, "128-byte-swizzled bias tiles need 1 KB alignment");

// Bounded wait on an mbarrier that also gives up once another role aborted.
// Warp-uniform when every lane of the warp calls it.
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

// Exponents (s*c^-1/2 + b)*log2e - m of 32 keys (raw S bits in u, keys
// 32*c32.. of the tile) of this thread's query row, in place; bias from the
// 128-byte-swizzled tile row in shared memory.
__device__ __forceinline__ void exponents32(uint32_t (&u)[32], const uint8_t *brow, int row,
                                            int c32, uint64_t c1x2, uint64_t l2e2,
                                            uint64_t nm2) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int ch = c32 * 4 + q;              // 16-byte chunk of 8 keys
    const uint4 bv = *reinterpret_cast<const uint4 *>(brow + ((ch ^ (row & 7)) << 4));
    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int jj = q * 8 + e * 2;
      const uint64_t bl = fma2(f2pack(bf16lo(bw[e]), bf16hi(bw[e])), l2e2, nm2);
      const float2 v =
          f2unpack(fma2(f2pack(__uint_as_float(u[jj]), __uint_as_float(u[jj + 1])), c1x2, bl));
      u[jj] = __float_as_uint(v.x);
      u[jj + 1] = __float_as_uint(v.y);
    }
  }
}

// Probabilities of 32 keys from their exponents: bf16 pairs into pk, running
// sums into sa/sb. MASKED: keys whose bit in mword is clear give 0. POLY > 0:
// every POLY-th key pair takes the FMA-pipe exp2 instead of the MUFU one.
template <bool MASKED, int POLY>
__device__ __forceinline__ void probs32(const uint32_t (&u)[32], uint32_t mword, uint64_t &sa,
                                        uint64_t &sb, uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float p0, p1;
    if (POLY > 0 && (e / 2) % POLY == POLY - 1) {
      const float2 pp =
          f2unpack(exp2_fma2(f2pack(__uint_as_float(u[e]), __uint_as_float(u[e + 1]))));
      p0 = pp.x;
      p1 = pp.y;
    } else {
      p0 = ex2_approx(__uint_as_float(u[e]));
      p1 = ex2_approx(__uint_as_float(u[e + 1]));
    }
    if (MASKED) {
      if (!((mword >> e) & 1u)) p0 = 0.0f;
      if (!((mword >> (e + 1)) & 1u)) p1 = 0.0f;
    }
    if (e & 2) sb = add2(sb, f2pack(p0, p1));
    else sa = add2(sa, f2pack(p0, p1));
    pk[e / 2] = kPackOnIntegerPipes ? pack_bf16_int(p0, p1) : pack_bf16(p0, p1);
  }
}

template <int POLY>
__global__ void __launch_bounds__(kThreads, 1)
fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_b,
                const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  FwdSmem &ctl = *reinterpret_cast<FwdSmem *>(smem + kOffCtl);
  volatile uint32_t *abort_flag = &ctl.abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = a.N;
  const int xb = blockIdx.x, h = blockIdx.y;
  const int r0 = a.row0 + blockIdx.z * kRows;   // row of the stacked problems
  const int nrows = min(kRows, a.row_end - r0);
  // problem of these rows and the first one's row inside it (N % 8 == 0, so the
  // 8 rows of a CTA belong to one problem)
  const int pb = r0 / N;
  const int rb0 = r0 - pb * N;
  const int nkb = (N + kBN - 1) / kBN;
  const int T = nkb * kRows;        // (key tile, row) steps, row fastest

  if (threadIdx.x == 0) {
    mbar_init(&ctl.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.kv_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl.bias_full[b], 1);
      mbar_init(&ctl.bias_empty[b], 128 * kGroups);
    }
    for (int w = 0; w < kGroups; ++w) {
      mbar_init(&ctl.s_full[w], 1);
      mbar_init(&ctl.p_full[w], 128);   // buffer w belongs to warpgroup w
    }
    for (int rr = 0; rr < kRows; ++rr) mbar_init(&ctl.o_done[rr], 1);
    mbar_init(&ctl.o_final, 1);
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
    if (elect_one() && nrows == kRows) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_b);
      int armed_kv[kStages];
      int armed_b[2] = {-1, -1};
      for (int s = 0; s < kStages; ++s) armed_kv[s] = -1;
      bool ok = true;
      mbar_arrive_expect_tx(&ctl.q_full, kRows * kQTileBytes);
      for (int rr = 0; rr < kRows; ++rr) {
        uint8_t *dst = smem + kOffQ + rr * kQTileBytes;
        if (a.x_inner)
          tma_load_5d(dst, &tm_q, &ctl.q_full, 0, h, xb * kBM, rb0 + rr, pb);
        else
          tma_load_5d(dst, &tm_q, &ctl.q_full, 0, h, rb0 + rr, xb * kBM, pb);
      }
      int it = 0;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int bb = kb & 1;
        if (kb >= 2 && !wait_bar(&ctl.bias_empty[bb], ((kb >> 1) - 1) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&ctl.bias_full[bb], kBiasTileBytes);
        tma_load_3d(smem + kOffB + bb * kBiasTileBytes, &tm_b, &ctl.bias_full[bb], kb * kBN,
                    xb * kBM, pb * a.H + h);
        armed_b[bb] = kb >> 1;
        for (int rr = 0; rr < kRows; ++rr, ++it) {
          const int st = it % kStages;
          if (it >= kStages &&
              !wait_bar(&ctl.kv_empty[st], ((it / kStages) - 1) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&ctl.kv_full[st], 2 * kKVTileBytes + 16);
          uint8_t *kd = smem + kOffK + st * kKVTileBytes;
          uint8_t *vd = smem + kOffV + st * kKVTileBytes;
          if (a.x_inner) {
            tma_load_5d(kd, &tm_k, &ctl.kv_full[st], 0, h, kb * kBN, rb0 + rr, pb);
            tma_load_5d(vd, &tm_v, &ctl.kv_full[st], 0, h, kb * kBN, rb0 + rr, pb);
          } else {
            tma_load_5d(kd, &tm_k, &ctl.kv_full[st], 0, h, rb0 + rr, kb * kBN, pb);
            tma_load_5d(vd, &tm_v, &ctl.kv_full[st], 0, h, rb0 + rr, kb * kBN, pb);
          }
          // the 4 key-bit words of the 128 keys around this tile (16-byte aligned)
          bulk_load(smem + kOffMask + st * 16,
                    a.mask_bits + (int64_t)(a.mask_per_row ? r0 + rr : pb) * a.mask_bits_stride +
                        (kb >> 1) * 4,
                    16,
                    &ctl.kv_full[st]);
          armed_kv[st] = it / kStages;
        }
      }
      if (!ok) {
        // Let every copy this thread started land before the CTA exits.
        mbar_wait(&ctl.q_full, 0);
        for (int s = 0; s < kStages; ++s)
          if (armed_kv[s] >= 0) mbar_wait(&ctl.kv_full[s], armed_kv[s] & 1);
        for (int b = 0; b < 2; ++b)
          if (armed_b[b] >= 0) mbar_wait(&ctl.bias_full[b], armed_b[b] & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (elect_one() && nrows == kRows) {
      const uint32_t id_s = make_idesc_bf16(kBM, kBN, false, false);
      const uint32_t id_pv = make_idesc_bf16(kBM, kC, false, true);
      bool ok = wait_bar(&ctl.q_full, 0, abort_flag, a.status);
      tc_fence_after();
      // S of step t into the S buffer of its warpgroup
      auto issue_s = [&](int t) -> bool {
        const int w = t % kGroups, rr = t % kRows, st = t % kStages;
        if (!wait_bar(&ctl.kv_full[st], (t / kStages) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t qa = smem_u32(smem + kOffQ + rr * kQTileBytes);
        const uint32_t ka = smem_u32(smem + kOffK + st * kKVTileBytes);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
          const uint64_t da = make_sdesc(qa + ks * 32, 16, 512, kSwizzle64B);
          const uint64_t db = make_sdesc(ka + ks * 32, 16, 512, kSwizzle64B);
          mma_ss(tmem + w * kBN, da, db, id_s, ks > 0 ? 1u : 0u);
        }
        mma_commit(&ctl.s_full[w]);
        return true;
      };
      // O[row] += P V of step t, P read from the warpgroup's S buffer
      auto issue_pv = [&](int t) -> bool {
        const int w = t % kGroups, rr = t % kRows, kb = t / kRows, st = t % kStages;
        if (!wait_bar(&ctl.p_full[w], (t / kGroups) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t va = smem_u32(smem + kOffV + st * kKVTileBytes);
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks) {
          const uint64_t db = make_sdesc(va + ks * 16 * 64, 512, 512, kSwizzle64B);
          mma_ts(tmem + kColO + rr * kC, tmem + w * kBN + ks * 8, db, id_pv,
                 (kb > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&ctl.kv_empty[st]);
        mma_commit(&ctl.o_done[rr]);
        return true;
      };
      // The PV product of step t - kGroups reads the S buffer that S of step t
      // overwrites, so it is issued first (the tensor pipe runs them in order).
      for (int t = 0; ok && t < T; ++t) {
        if (t >= kGroups) ok = issue_pv(t - kGroups);
        if (ok) ok = issue_s(t);
      }
      for (int t = max(0, T - kGroups); ok && t < T; ++t) ok = issue_pv(t);
      mma_commit(&ctl.o_final);
      // No tensor-memory operation may be in flight when the CTA tears down.
      mma_commit(&ctl.teardown);
      mbar_wait(&ctl.teardown, 0);
    }
  } else {
    // ------------------------------------------------ softmax and epilogue --
    const int wg = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;           // query within the tile = TMEM lane
    const int x = xb * kBM + row;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t sbuf = tl + wg * kBN;
    const uint64_t c1x2 = f2pack(a.scale * kLog2e, a.scale * kLog2e);
    const uint64_t l2e2 = f2pack(kLog2e, kLog2e);
    // running max and sum of this warpgroup's two rows (rows wg and wg + 4); the
    // loop over them is not unrolled, so the pair swaps instead of being indexed
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.0f, 0.0f};
    auto swap_rows = [&]() {
      const float m0 = m_r[0], l0 = l_r[0];
      m_r[0] = m_r[1];
      l_r[0] = l_r[1];
      m_r[1] = m0;
      l_r[1] = l0;
    };
    bool ok = nrows == kRows;
    if (!ok) {
      *abort_flag = 1u;
      report_status(a.status, kStatusBounds);
    }
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int bb = kb & 1;
      if (!wait_bar_warp(&ctl.bias_full[bb], (kb >> 1) & 1, abort_flag, a.status)) {
        ok = false;
        break;
      }
      const uint8_t *brow = smem + kOffB + bb * kBiasTileBytes + row * 128;
      // max of this query row's 64 bias values (shared by all rows of the CTA)
      float bmax = -INFINITY;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint4 bv = *reinterpret_cast<const uint4 *>(brow + ((ch ^ (row & 7)) << 4));
        bmax = fmax3(bmax, fmax3(bf16lo(bv.x), bf16hi(bv.x), bf16lo(bv.y)),
                     fmax3(bf16hi(bv.y), fmax3(bf16lo(bv.z), bf16hi(bv.z), bf16lo(bv.w)),
                           bf16hi(bv.w)));
      }
#pragma unroll 1
      for (int j = 0; j < 2; ++j, swap_rows()) {
        const int rr = wg + kGroups * j;
        const int it = kb * kRows + rr;
        const int st = it % kStages;
        // key bits of this row and key tile arrive with the K/V stage
        if (!wait_bar_warp(&ctl.kv_full[st], (it / kStages) & 1, abort_flag, a.status) ||
            !wait_bar_warp(&ctl.s_full[wg], (it / kGroups) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        const uint4 mw = *reinterpret_cast<const uint4 *>(smem + kOffMask + st * 16);
        const uint32_t mk0 = (kb & 1) ? mw.z : mw.x, mk1 = (kb & 1) ? mw.w : mw.y;
        const bool full_tile = (mk0 & mk1) == 0xffffffffu;
        tc_fence_after();
        // Pass 1: an upper bound of the row's logits, max(s) * c^-1/2 + max(b).
        // Softmax is exact for any shift; a bound keeps every exponent <= 0.
        float sm0 = -INFINITY, sm1 = -INFINITY;
        {
          uint32_t u[32], w[32];
          tmem_ld32x2(sbuf, sbuf + 32, u, w);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            sm0 = fmax3(sm0, __uint_as_float(u[e]), __uint_as_float(u[e + 1]));
            sm1 = fmax3(sm1, __uint_as_float(w[e]), __uint_as_float(w[e + 1]));
          }
        }
        // log2-domain bound; the running max only moves when the bound grows by
        // more than 8, so most tiles skip the rescale of O (p stays <= 2^8).
        const float bound = (fmaxf(sm0, sm1) * a.scale + bmax) * kLog2e;
        const float m_old = m_r[0];
        const float m_new = bound > m_old + 8.0f ? bound : m_old;
        const float alpha = ex2_approx(m_old - m_new);   // m_old = -inf gives 0
        const uint64_t nm2 = f2pack(-m_new, -m_new);
        uint64_t sum_a = 0, sum_b = 0;   // two packed running sums (bit pattern 0 = 0.0f)
#pragma unroll 1
        for (int c32 = 0; c32 < 2; ++c32) {
          uint32_t u[32];
          uint32_t pk[16];
          tmem_ld32(sbuf + 32 * c32, u);
          // P (bf16 pairs) of keys 32*c32.. goes to columns 16*c32.. of this S
          // buffer, whose S values were already read into registers.
          exponents32(u, brow, row, c32, c1x2, l2e2, nm2);
          if (full_tile) probs32<false, POLY>(u, c32 ? mk1 : mk0, sum_a, sum_b, pk);
          else probs32<true, POLY>(u, c32 ? mk1 : mk0, sum_a, sum_b, pk);
          tmem_st16(sbuf + 16 * c32, pk);
        }
        const float2 sa = f2unpack(add2(sum_a, sum_b));
        l_r[0] = l_r[0] * alpha + (sa.x + sa.y);
        m_r[0] = m_new;
        if (kb > 0) {
          // rescale the running output once the previous PV of this row is done
          if (!wait_bar_warp(&ctl.o_done[rr], (kb - 1) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (__any_sync(0xffffffffu, alpha != 1.0f)) {
            uint32_t o[32];
            const uint32_t oa = tl + kColO + rr * kC;
            tmem_ld32(oa, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(oa, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&ctl.p_full[wg]);
      }
      if (ok) mbar_arrive(&ctl.bias_empty[bb]);
    }
    // epilogue: out = sigmoid(g) * O / l (bf16), lse = ln(sum exp s)
    if (ok) ok = wait_bar_warp(&ctl.o_final, 0, abort_flag, a.status);
    if (ok) tc_fence_after();
#pragma unroll 1
    for (int j = 0; j < 2; ++j, swap_rows()) {
      const int rr = wg + kGroups * j;
      const int r = r0 + rr;
      uint32_t o[32];
      if (ok) tmem_ld32(tl + kColO + rr * kC, o);
      if (x >= N || rr >= nrows) continue;
      float *lse_p = a.lse + ((int64_t)r * a.H + h) * N + x;
      if (!ok) {
        *lse_p = __int_as_float(0x7fc00000);  // NaN marks a tile the kernel gave up on
        continue;
      }
      const float l = l_r[0];
      const float inv = l > 0.0f ? rcp_approx(l) : 0.0f;
      const int64_t off = (int64_t)pb * N * N * a.H * kC + (int64_t)(rb0 + rr) * a.sR +
                          (int64_t)x * a.sX + (int64_t)h * kC;
      const uint4 *gp = reinterpret_cast<const uint4 *>(a.gate + off);
      uint4 *op = reinterpret_cast<uint4 *>(a.out + off);
      uint4 *rp = a.out_res ? reinterpret_cast<uint4 *>(a.out_res + off) : nullptr;
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        const uint4 gv = gp[v4];
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
        uint32_t ow[4], rw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int cc = v4 * 8 + e * 2;
          const float g0 = bf16lo(gw[e]), g1 = bf16hi(gw[e]);
          const float s0 = rcp_approx(1.0f + ex2_approx(-g0 * kLog2e));
          const float s1 = rcp_approx(1.0f + ex2_approx(-g1 * kLog2e));
          const float y0 = s0 * __uint_as_float(o[cc]) * inv;
          const float y1 = s1 * __uint_as_float(o[cc + 1]) * inv;
          ow[e] = pack_bf16(y0, y1);
          // what the bf16 output lost, itself kept to bf16 precision
          rw[e] = pack_bf16(y0 - bf16lo(ow[e]), y1 - bf16hi(ow[e]));
        }
        op[v4] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        if (rp) rp[v4] = make_uint4(rw[0], rw[1], rw[2], rw[3]);
      }
      *lse_p = l > 0.0f ? (m_r[0] + lg2_approx(l)) * kLn2 : -INFINITY;
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

int fwd_bf16_rows_per_cta() { return kRows; }
int fwd_bf16_key_tile() { return kBN; }

template <int POLY>
cudaError_t launch_fwd_poly(const FwdMaps &maps, const FwdArgs &args, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(fwd_bf16_kernel<POLY>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((args.N + kBM - 1) / kBM, args.H, (args.row_end - args.row0 + kRows - 1) / kRows);
  fwd_bf16_kernel<POLY><<<grid, kThreads, kSmemBytes, stream>>>(maps.q, maps.k, maps.v,
                                                                 maps.bias, args);
  return cudaGetLastError();
}

cudaError_t launch_fwd_bf16(const FwdMaps &maps, const FwdArgs &args, cudaStream_t stream) {
  if (args.N == 0) return cudaSuccess;
  // the exp2 split: one key pair in four on the FMA pipe
  return args.exp2_split ? launch_fwd_poly<4>(maps, args, stream)
                         : launch_fwd_poly<0>(maps, args, stream);
}

}  // namespace tri
