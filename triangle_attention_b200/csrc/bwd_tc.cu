// bf16 backward of gated triangle self-attention on sm_100a with every
// cross-tile gradient sum on chip (tcgen05 + TMA + an L2-resident exchange).
//
// Work unit: one CTA owns one (query tile X, key tile Y, head h) block of the
// probability matrix and walks all attention rows of its row group in order.
// For every row it recomputes the 128x128 block of probabilities once from the
// saved log-sum-exp and reuses it for all four gradients ("TurboPairFormer
// accelera fino a 1,73x l'addestramento di OpenFold3 nei test", section "Dove si
// impiega il tempo"). The block is held transposed, keys on tensor-memory lanes:
//   S^T  = K Q^T,  dP^T = V dU^T                   (tcgen05, tensor memory)
//   P^T  = exp(S^T c^-1/2 + b - lse), dS^T = P^T (dP^T - D)   (16 warps)
//   dV_t = P^T dU, dK_t = dS^T Q  (A operand read from tensor memory)
//   dQ_t = dS K                   (A operand: dS^T written to shared memory)
//   dbias[h, X, Y] += dS          (fp32 registers, every row of the group)
//
// The pair-bias gradient block stays in registers for the whole row walk, so
// its sum over the rows runs in one fixed order. Each row's dq block still has
// to be summed over the key tiles and its dk/dv blocks over the query tiles:
// the CTA drains its three gradient blocks from tensor memory (rounded to bf16)
// into a small ring in global memory that stays in L2 (a few rows deep), and for
// every (row, output tile) one owner CTA of the same grid sums the contributions
// in tile order in fp32 and rounds the result to bf16 once. Readiness and reuse of ring slots travel through
// integer flags with release/acquire ordering; there are no floating-point
// atomics, so repeated calls are bit-identical. All CTAs that exchange blocks
// are resident at once (at most one CTA per SM, no more CTAs than SMs).
//
// Warp roles (640 threads):
//   warp 0      tensor-memory allocator and MMA issuer; publishes each row's
//               exported gradient blocks
//   warp 1      TMA producer: Q, dU, K, V tiles, the lse/D pairs and the key
//               mask bits of each row
//   warps 2, 3  owner-side sums: bulk copies of the ring contributions into
//               shared memory, fixed-order fp32 sums, bf16 results (the two
//               warps take alternate blocks of an owned row)
//   warps 4..19 four elementwise warpgroups; warpgroup g handles the queries
//               32g .. 32g+31 of the block for all 128 keys (thread = key lane)
//               and, once a row's gradient MMAs are done, drains channels
//               8g .. 8g+7 of its dq, dk and dv blocks into the ring
//
// Tensor memory: buffer b (row & 1) at columns 256*b: S^T at +0..127, dP^T at
// +128..255. The elementwise warps overwrite the S^T columns of each 16-query
// chunk with that chunk's P^T (bf16 pairs, 8 columns) and dS^T (8 columns), so
// the operands of MMA K-step ks sit at +16*ks (P^T) and +16*ks+8 (dS^T). The
// gradient blocks then land in the consumed dP^T columns: dQ at +128, dK at
// +160, dV at +192. Tensor-pipe order per row t: dQ(t), dK(t), dV(t), S^T(t+2)
// into the same buffer (the pipe runs them in order, so S^T(t+2) overwrites
// P^T/dS^T only after dK/dV have read them), then, once the elementwise
// warps have drained the gradient blocks of row t (in the middle of row t+1),
// dP^T(t+2).
#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>

#include "bf16.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace tri {
namespace {

constexpr int kT = 128;                       // queries per tile = keys per tile
constexpr int kC = 32;
constexpr int kStages = 3;                    // input stages (rows in flight)
constexpr int kRing = 8;                      // ring slots (rows between export and sum)
constexpr int kMaxStg = 8;                    // owner-side staging buffers at most
constexpr int kMmaWarp = 0;
constexpr int kLoadWarp = 1;
constexpr int kReduceWarp = 2;                // and kReduceWarp + 1
constexpr int kReduceWarps = 2;
constexpr int kEltWarp0 = 4;
constexpr int kEltWarps = 16;
constexpr int kThreads = (kEltWarp0 + kEltWarps) * 32;
constexpr int kEltThreads = kEltWarps * 32;
constexpr int kMaxNb = 12;                    // tiles per axis this kernel takes
// The ring holds a gradient block channel-group-major, [4][128 lanes][8]; an
// owner-side sum block is 64 lanes of one channel group (1 KB per contribution).
constexpr int kRedLanes = 64;
constexpr int kRedBlocks = 4 * (kT / kRedLanes);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBufCols = 256;
constexpr uint32_t kColS = 0, kColDP = 128, kColGQ = 128, kColGK = 160, kColGV = 192;
constexpr uint32_t kTileBytes = kT * kC * 2;               // 8 KB pair tile
constexpr uint32_t kSqBytes = kT * kT * 2;                 // 32 KB
constexpr uint32_t kStageBytes = 4 * kTileBytes;           // Q, dU, K, V
constexpr uint32_t kLDBytes = kT / 2 * 16;                 // 64 (lse, D) pairs: 1 KB
constexpr uint32_t kRowBytes = kLDBytes + 16;              // + 4 key-mask words
constexpr uint32_t kBlkBytes = kRedLanes * 8 * 2;          // 1 KB per contribution block
constexpr uint32_t kGradElems = kT * kC;                   // one gradient block
// Shared memory (1 KB-aligned base):
constexpr uint32_t kOffIn = 0;                                        // stages
constexpr uint32_t kOffDS = kOffIn + kStages * kStageBytes;           // 2 dS tiles
constexpr uint32_t kOffBias = kOffDS + 2 * kSqBytes;                  // bias[key][query]
constexpr uint32_t kOffStg = kOffBias + kSqBytes;                     // owner-side staging
constexpr uint32_t kStgBytes = 24 * 1024;
constexpr uint32_t kOffRow = kOffStg + kStgBytes;                     // row blocks
constexpr uint32_t kOffCtl = kOffRow + kStages * kRowBytes;
constexpr float kLog2e = 1.4426950408889634f;

static_assert(kOffDS % 1024 == 0 && kOffBias % 1024 == 0 && kOffStg % 1024 == 0,
              "tiles need 1 KB alignment");
static_assert(kOffCtl % 8 == 0, "barriers need 8-byte alignment");

struct __align__(8) Ctl {
  uint64_t in_full[kStages];
  uint64_t in_empty[kStages];
  uint64_t sdp_full[2];      // S^T and dP^T of the row in TMEM buffer b are ready
  uint64_t pds_full[2];      // P^T/dS^T (TMEM buffer b) and dS (SMEM tile b) are written
  uint64_t pds_free[2];      // dQ has read dS tile b
  uint64_t gv_done[2];       // dQ, dK, dV blocks in TMEM buffer b complete
  uint64_t drained[2];       // the elementwise warps have moved them to the ring
  uint64_t stg_full[kMaxStg];  // owner-side staging buffer s filled
  uint64_t teardown;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

constexpr uint32_t kSmemBytes = kOffCtl + sizeof(Ctl);
static_assert(kSmemBytes <= 227u * 1024u, "over the per-block shared memory limit");

__device__ __forceinline__ bool aborted(volatile uint32_t *f) { return *f != 0u; }

__device__ __forceinline__ void fail(volatile uint32_t *abort_flag, int32_t *status,
                                     int32_t code) {
  *abort_flag = 1u;
  report_status(status, code);
}

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
  fail(abort_flag, status, kStatusTimeout);
  return false;
}

__device__ __forceinline__ bool wait_bar_warp(uint64_t *bar, uint32_t parity,
                                              volatile uint32_t *abort_flag, int32_t *status) {
  const bool ok = wait_bar(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait until the GPU-scope flag reaches `target` (acquire).
__device__ __forceinline__ bool wait_flag(const int32_t *flag, int32_t target,
                                          volatile uint32_t *abort_flag, int32_t *status) {
  if (ld_acquire_gpu(flag) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t polls = 1; polls < kWaitMaxPolls; ++polls) {
    if (ld_acquire_gpu(flag) >= target) return true;
    if ((polls & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
    }
  }
  fail(abort_flag, status, kStatusTimeout);
  return false;
}

// 16 bytes (8 bf16) into a 128x128 tile laid out as two 128-row x 128-byte
// halves with the 128-byte swizzle (chunk ^= row & 7).
__device__ __forceinline__ void st_tile_chunk(uint8_t *tile, int row, int half, int chunk,
                                              uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  uint8_t *p = tile + half * (kSqBytes / 2) + row * 128 + ((chunk ^ (row & 7)) << 4);
  *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}

// Ring address of gradient block `type` (0 dq, 1 dk, 2 dv) of output tile
// `out`, contribution `con`, in slot `slot` of local (group, head) pair z; the
// block is [4 channel groups][128 lanes][8 channels] in bf16.
__device__ __forceinline__ __nv_bfloat16 *ring_block(const BwdTcArgs &a, int slot, int z,
                                                     int type, int out, int con) {
  const int64_t blk = ((((int64_t)slot * a.ghl + z) * 3 + type) * a.nb + out) * a.nb + con;
  return a.ring + blk * kGradElems;
}

__global__ void __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_du,
              const BwdTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    // the layout has no room for realignment: refuse rather than misplace tiles
    if (threadIdx.x == 0) report_status(a.status, kStatusBounds);
    return;
  }
  Ctl &ctl = *reinterpret_cast<Ctl *>(smem + kOffCtl);
  volatile uint32_t *abort_flag = &ctl.abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = a.N, H = a.H, nb = a.nb;
  const int X = blockIdx.x, Y = blockIdx.y, z = blockIdx.z;
  const int gh = a.gh0 + z;
  const int g = gh / H, h = gh % H;
  const int r0 = g * a.rows_per_group;
  const int r1 = min(N, r0 + a.rows_per_group);
  const int T = max(0, r1 - r0);
  // flags of this (group, head) pair
  int32_t *exported = a.exported + (int64_t)gh * nb * nb;
  int32_t *cons_q = a.consumed_q + (int64_t)gh * nb * kRing * kReduceWarps;
  int32_t *cons_kv = a.consumed_kv + (int64_t)gh * nb * kRing * kReduceWarps;

  // Tensor memory first, while warp 0 is still converged (the allocation is a
  // .sync.aligned warp instruction); warp 3 sets up the barriers meanwhile.
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 3 * 32) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.in_full[s], 1);
      mbar_init(&ctl.in_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl.sdp_full[b], 1);
      mbar_init(&ctl.pds_full[b], kEltThreads);
      mbar_init(&ctl.pds_free[b], 1);
      mbar_init(&ctl.gv_done[b], 1);
      mbar_init(&ctl.drained[b], kEltThreads);
    }
    for (int b = 0; b < kMaxStg; ++b) mbar_init(&ctl.stg_full[b], 1);
    mbar_init(&ctl.teardown, 1);
    ctl.abort_flag = 0u;
    fence_barrier_init();
  }
  // lse/D pairs past the last query of a ragged tile: -inf exponent (p = 0) and D = 0
  const int xvalid = min(kT, N - X * kT);
  for (int i = threadIdx.x; i < kStages * (kT / 2); i += kThreads) {
    const int s = i / (kT / 2), pr = i % (kT / 2);
    if (2 * pr >= xvalid)
      *reinterpret_cast<float4 *>(smem + kOffRow + s * kRowBytes + pr * 16) =
          make_float4(-INFINITY, -INFINITY, 0.0f, 0.0f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == kMmaWarp || warp == kLoadWarp) {
    // ----------------------------------------- MMA issue (0), loads (1) --
    const bool mma_lane = warp == kMmaWarp && lane == 0;
    const bool load_lane = warp == kLoadWarp && lane == 0;
    const uint32_t id_s = make_idesc_bf16(kT, kT, false, false);
    const uint32_t id_q = make_idesc_bf16(kT, kC, true, true);
    const uint32_t id_t = make_idesc_bf16(kT, kC, false, true);
    const uint32_t lse_bytes = (uint32_t)(xvalid / 2) * 16u;

    auto stage_addr = [&](int t) { return smem_u32(smem + kOffIn + (t % kStages) * kStageBytes); };
    auto issue_st = [&](int t) {          // S^T(t) = K Q^T into buffer t & 1
      const uint32_t in = stage_addr(t);
      const uint32_t qa = in, ka = in + 2 * kTileBytes;
      const uint32_t d = tmem + (t & 1) * kBufCols + kColS;
#pragma unroll
      for (int ks = 0; ks < kC / 16; ++ks)
        mma_ss(d, make_sdesc(ka + ks * 32, 16, 512, kSwizzle64B),
               make_sdesc(qa + ks * 32, 16, 512, kSwizzle64B), id_s, ks > 0 ? 1u : 0u);
    };
    auto issue_dpt = [&](int t) {         // dP^T(t) = V dU^T, then mark S^T/dP^T ready
      const uint32_t in = stage_addr(t);
      const uint32_t ua = in + kTileBytes, va = in + 3 * kTileBytes;
      const uint32_t d = tmem + (t & 1) * kBufCols + kColDP;
#pragma unroll
      for (int ks = 0; ks < kC / 16; ++ks)
        mma_ss(d, make_sdesc(va + ks * 32, 16, 512, kSwizzle64B),
               make_sdesc(ua + ks * 32, 16, 512, kSwizzle64B), id_s, ks > 0 ? 1u : 0u);
      mma_commit(&ctl.sdp_full[t & 1]);
    };
    auto issue_grads = [&](int t) {
      const int b = t & 1;
      const uint32_t in = stage_addr(t);
      const uint32_t qa = in, ua = in + kTileBytes, ka = in + 2 * kTileBytes;
      const uint32_t dsa = smem_u32(smem + kOffDS + b * kSqBytes);
      const uint32_t tb = tmem + b * kBufCols;
      // dQ = dS K: A = dS (queries x keys) read MN-major from the [key][query]
      // tile, B = K (keys x c) read MN-major; K-step = 16 keys
#pragma unroll
      for (int ks = 0; ks < kT / 16; ++ks)
        mma_ss(tb + kColGQ, make_sdesc(dsa + ks * 2048, kSqBytes / 2, 1024, kSwizzle128B),
               make_sdesc(ka + ks * 1024, 512, 512, kSwizzle64B), id_q, ks > 0 ? 1u : 0u);
      mma_commit(&ctl.pds_free[b]);
      // dK = dS^T Q and dV = P^T dU: A from tensor memory, K-step = 16 queries
#pragma unroll
      for (int ks = 0; ks < kT / 16; ++ks)
        mma_ts(tb + kColGK, tb + kColS + 16 * ks + 8,
               make_sdesc(qa + ks * 1024, 512, 512, kSwizzle64B), id_t, ks > 0 ? 1u : 0u);
#pragma unroll
      for (int ks = 0; ks < kT / 16; ++ks)
        mma_ts(tb + kColGV, tb + kColS + 16 * ks,
               make_sdesc(ua + ks * 1024, 512, 512, kSwizzle64B), id_t, ks > 0 ? 1u : 0u);
      mma_commit(&ctl.gv_done[b]);
      mma_commit(&ctl.in_empty[t % kStages]);
    };

    if (mma_lane && T > 0) {
      bool ok = true;
      for (int t = 0; ok && t < min(2, T); ++t) {
        ok = wait_bar(&ctl.in_full[t % kStages], (t / kStages) & 1, abort_flag, a.status);
        if (ok) {
          tc_fence_after();
          issue_st(t);
          issue_dpt(t);
        }
      }
      for (int t = 0; ok && t < T; ++t) {
        const int b = t & 1;
        ok = wait_bar(&ctl.pds_full[b], (t >> 1) & 1, abort_flag, a.status);
        if (!ok) break;
        tc_fence_after();
        issue_grads(t);
        if (t + 2 < T) {
          ok = wait_bar(&ctl.in_full[(t + 2) % kStages], ((t + 2) / kStages) & 1, abort_flag,
                        a.status);
          if (!ok) break;
          tc_fence_after();
          issue_st(t + 2);
        }
        // the gradient blocks of row t have left tensor memory for the ring
        ok = wait_bar(&ctl.drained[b], (t >> 1) & 1, abort_flag, a.status);
        if (!ok) break;
        // the drains' ring stores (observed through the barrier) precede this release
        st_release_gpu(exported + X * nb + Y, t + 1);
        if (t + 2 < T) {
          tc_fence_after();
          issue_dpt(t + 2);
        }
      }
      // No tensor-memory operation may be in flight when the CTA tears down.
      mma_commit(&ctl.teardown);
      mbar_wait(&ctl.teardown, 0);
    }
    if (load_lane && T > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_du);
      // per stage: 1 + the phase its last copies complete, 0 if never used
      uint32_t armed0 = 0u, armed1 = 0u, armed2 = 0u;
      static_assert(kStages == 3, "armed phases are kept for three stages");
      bool ok = true;
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % kStages, r = r0 + t;
        if (t >= kStages &&
            !wait_bar(&ctl.in_empty[st], ((t / kStages) - 1) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        uint8_t *in = smem + kOffIn + st * kStageBytes;
        uint8_t *rb = smem + kOffRow + st * kRowBytes;
        mbar_arrive_expect_tx(&ctl.in_full[st], kStageBytes + lse_bytes + 16);
        if (a.x_inner) {
          tma_load_5d(in, &tm_q, &ctl.in_full[st], 0, h, X * kT, r, 0);
          tma_load_5d(in + 2 * kTileBytes, &tm_k, &ctl.in_full[st], 0, h, Y * kT, r, 0);
          tma_load_5d(in + 3 * kTileBytes, &tm_v, &ctl.in_full[st], 0, h, Y * kT, r, 0);
        } else {
          tma_load_5d(in, &tm_q, &ctl.in_full[st], 0, h, r, X * kT, 0);
          tma_load_5d(in + 2 * kTileBytes, &tm_k, &ctl.in_full[st], 0, h, r, Y * kT, 0);
          tma_load_5d(in + 3 * kTileBytes, &tm_v, &ctl.in_full[st], 0, h, r, Y * kT, 0);
        }
        tma_load_5d(in + kTileBytes, &tm_du, &ctl.in_full[st], 0, h, X * kT, r, 0);
        bulk_load(rb, a.LD + ((int64_t)r * H + h) * (N / 2) + X * (kT / 2), lse_bytes,
                  &ctl.in_full[st]);
        bulk_load(rb + kLDBytes, a.mask_bits + (int64_t)r * a.mask_bits_stride + Y * 4, 16,
                  &ctl.in_full[st]);
        const uint32_t ph = 1u + ((t / kStages) & 1);
        if (st == 0) armed0 = ph;
        else if (st == 1) armed1 = ph;
        else armed2 = ph;
        // ask L2 for the tiles of a row further ahead
        const int rp = r + kStages + 1;
        if (rp < r1) {
          if (a.x_inner) {
            tma_prefetch_l2_5d(&tm_q, 0, h, X * kT, rp, 0);
            tma_prefetch_l2_5d(&tm_k, 0, h, Y * kT, rp, 0);
            tma_prefetch_l2_5d(&tm_v, 0, h, Y * kT, rp, 0);
          } else {
            tma_prefetch_l2_5d(&tm_q, 0, h, rp, X * kT, 0);
            tma_prefetch_l2_5d(&tm_k, 0, h, rp, Y * kT, 0);
            tma_prefetch_l2_5d(&tm_v, 0, h, rp, Y * kT, 0);
          }
          tma_prefetch_l2_5d(&tm_du, 0, h, X * kT, rp, 0);
        }
      }
      // every copy this thread started lands before the CTA exits
      if (armed0) mbar_wait(&ctl.in_full[0], armed0 - 1);
      if (armed1) mbar_wait(&ctl.in_full[1], armed1 - 1);
      if (armed2) mbar_wait(&ctl.in_full[2], armed2 - 1);
    }
  } else if (warp == kReduceWarp || warp == kReduceWarp + 1) {
    // ---------------------------------------- owner-side sums (warps 2, 3) --
    // Row u's dq block of query tile X is summed by CTA (X, u mod nb), its dk
    // and dv blocks of key tile Y by CTA ((u + nb/2) mod nb, Y): each CTA owns
    // one of each kind every nb rows. An owned row's blocks (8 per gradient
    // kind: 64 lanes x 8 channels, nb bf16 contributions each) alternate between
    // the two warps; each warp streams its blocks through its own `nstg`
    // staging buffers, all of them in flight at once, and marks the ring slot
    // consumed with its own flag.
    const int rw = warp - kReduceWarp;
    const uint32_t half = kStgBytes / kReduceWarps;
    const int nstg = min(kMaxStg / kReduceWarps, (int)(half / ((uint32_t)nb * kBlkBytes)));
    uint8_t *const stg_base = smem + kOffStg + rw * half;
    uint64_t *const stg_bar = &ctl.stg_full[rw * (kMaxStg / kReduceWarps)];
    uint32_t stg_phase = 0u;     // bit s: parity of the next completion of buffer s
    uint32_t stg_busy = 0u;      // bit s: a fill of buffer s is in flight
    bool ok = true;
    for (int u = 0; ok && u < T; ++u) {
      const bool own_q = (u % nb) == Y;
      const bool own_kv = ((u + nb / 2) % nb) == X;
      if (!own_q && !own_kv) continue;
      const int r = r0 + u;
      {
        // lane c waits for contributor c's dq block, lane 16 + c for its dk/dv blocks
        const int c = lane & 15;
        const bool kv = lane >= 16;
        bool mine = true;
        if (c < nb && (kv ? own_kv : own_q))
          mine = wait_flag(kv ? exported + c * nb + Y : exported + X * nb + c, u + 1,
                           abort_flag, a.status);
        ok = __all_sync(0xffffffffu, mine);
      }
      if (!ok) break;
      // the acquired contributions are read next by bulk copies (async proxy)
      if (lane == 0) fence_proxy_async_global();
      __syncwarp();
      const int type0 = own_q ? 0 : 1;
      const int nblk = ((own_kv ? 3 : 1) - type0) * kRedBlocks;
      const int nmine = (nblk - rw + kReduceWarps - 1) / kReduceWarps;
      // this warp's block i is block j = 2i + rw of the row: gradient kind
      // type0 + j / 8, channel group (j % 8) >> 1, lanes 64 * (j & 1) .. of
      // every contribution, into buffer i % nstg
      auto issue = [&](int i) {
        const int s = i % nstg;
        stg_busy |= 1u << s;
        if (lane == 0) {
          const int j = kReduceWarps * i + rw;
          const int type = type0 + j / kRedBlocks, k = j % kRedBlocks;
          const __nv_bfloat16 *src = ring_block(a, u % kRing, z, type, type == 0 ? X : Y, 0) +
                                     (k >> 1) * (kT * 8) + (k & 1) * (kRedLanes * 8);
          uint8_t *stg = stg_base + s * nb * kBlkBytes;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&stg_bar[s], nb * kBlkBytes);
          for (int c = 0; c < nb; ++c)
            bulk_load(stg + c * kBlkBytes, src + (int64_t)c * kGradElems, kBlkBytes, &stg_bar[s]);
        }
      };
      for (int i = 0; i < min(nstg, nmine); ++i) issue(i);
      for (int i = 0; ok && i < nmine; ++i) {
        const int j = kReduceWarps * i + rw, s = i % nstg;
        const int type = type0 + j / kRedBlocks, k = j % kRedBlocks;
        const int cg = k >> 1, out = type == 0 ? X : Y;
        ok = wait_bar_warp(&stg_bar[s], (stg_phase >> s) & 1u, abort_flag, a.status);
        if (!ok) break;
        stg_phase ^= 1u << s;
        stg_busy &= ~(1u << s);
        const uint8_t *stg = stg_base + s * nb * kBlkBytes;
        __nv_bfloat16 *dst = type == 0 ? a.dq : type == 1 ? a.dk : a.dv;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          // lane il of the 64-lane block: its 8 channels of every contribution,
          // summed in tile order in fp32; four contributions' loads in flight
          const int il = lane + 32 * m;
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};   // fp32 channel pairs
          for (int c0 = 0; c0 < nb; c0 += 4) {
            uint4 v[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              if (c0 + cc < nb)
                v[cc] = *reinterpret_cast<const uint4 *>(stg + (c0 + cc) * kBlkBytes + il * 16);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              if (c0 + cc < nb) {
                const uint32_t vw[4] = {v[cc].x, v[cc].y, v[cc].z, v[cc].w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  acc[e] = add2(acc[e], f2pack(bf16lo(vw[e]), bf16hi(vw[e])));
              }
          }
          const int xi = out * kT + (k & 1) * kRedLanes + il;   // query or key of the result
          if (xi < N) {
            const float f = type == 2 ? 1.0f : a.scale;
            const uint64_t f2 = f2pack(f, f);
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 w2 = f2unpack(mul2(acc[e], f2));
              o[e] = pack_bf16(w2.x, w2.y);
            }
            *reinterpret_cast<uint4 *>(dst + (int64_t)r * a.sR + (int64_t)xi * a.sX +
                                       (int64_t)h * kC + cg * 8) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        __syncwarp();
        if (i + nstg < nmine) issue(i + nstg);
      }
      // every bulk copy of this warp out of the ring slot has landed
      if (ok && lane == 0) {
        if (own_q) st_release_gpu(cons_q + (X * kRing + u % kRing) * kReduceWarps + rw, u + 1);
        if (own_kv) st_release_gpu(cons_kv + (Y * kRing + u % kRing) * kReduceWarps + rw, u + 1);
      }
      if (aborted(abort_flag)) ok = false;
    }
    // after a failure, the fills still in flight land before the CTA exits
    if (lane == 0)
      for (int s = 0; s < nstg; ++s)
        if ((stg_busy >> s) & 1u) mbar_wait(&stg_bar[s], (stg_phase >> s) & 1u);
  } else if (warp >= kEltWarp0) {
    // ----------------------------------------- elementwise (warps 4..19) --
    const int eg = (warp - kEltWarp0) >> 2;           // queries 32*eg .. 32*eg + 31
    const int q4 = warp & 3;
    const int key = q4 * 32 + lane;                   // key of the block = TMEM lane
    const int y = Y * kT + key;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const int jbase = 32 * eg;
    const uint64_t c1x2 = f2pack(a.scale * kLog2e, a.scale * kLog2e);
    const uint64_t l2e2 = f2pack(kLog2e, kLog2e);
    const bool shared_mask = a.mask_bits_stride == 0;
    // this thread's bias row b[x, y] for its 32 queries, in shared memory
    // (bias[key][query], 16-byte chunks swizzled by key & 7); a key past N, or
    // one the shared mask drops, gets -inf so every probability of it is 0
    bool key_live = y < N;
    if (key_live && shared_mask)
      key_live = (a.mask_bits[y >> 5] >> (y & 31)) & 1u;
    uint8_t *brow = smem + kOffBias + key * 256;
    const int64_t hb = (int64_t)h * N * N;
#pragma unroll 1
    for (int c8 = 0; c8 < 4; ++c8) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v0 = -INFINITY, v1 = -INFINITY;
        const int x0 = X * kT + jbase + 8 * c8 + 2 * e;
        if (key_live) {
          v0 = x0 < N ? __bfloat162float(a.bias[hb + (int64_t)x0 * a.bX + (int64_t)y * a.bY])
                      : 0.0f;
          v1 = x0 + 1 < N
                   ? __bfloat162float(a.bias[hb + (int64_t)(x0 + 1) * a.bX + (int64_t)y * a.bY])
                   : 0.0f;
        }
        w[e] = pack_bf16(v0, v1);
      }
      const int ch = (jbase >> 3) + c8;
      *reinterpret_cast<uint4 *>(brow + ((ch ^ (key & 7)) << 4)) = make_uint4(w[0], w[1], w[2],
                                                                              w[3]);
    }
    uint64_t db2[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) db2[e] = 0ull;

    // Channels 8*eg .. 8*eg+7 of the dq, dk and dv blocks of row t (TMEM buffer
    // t & 1, lanes of this warp) into the ring, then a mark that this thread is
    // done with them. Ring blocks are [4 channel groups][128 lanes][8], so a
    // warp's stores cover 512 contiguous bytes per block.
    auto drain = [&](int t) -> bool {
      bool free_slot = true;
      if (lane < 2 * kReduceWarps && t >= kRing) {
        // row t - kRing summed by both owner warps of both kinds: one flag per lane
        const int32_t need = t - kRing + 1;
        const int rwl = lane % kReduceWarps;
        free_slot = lane < kReduceWarps
                        ? wait_flag(cons_q + (X * kRing + t % kRing) * kReduceWarps + rwl, need,
                                    abort_flag, a.status)
                        : wait_flag(cons_kv + (Y * kRing + t % kRing) * kReduceWarps + rwl, need,
                                    abort_flag, a.status);
      }
      if (!__all_sync(0xffffffffu, free_slot)) return false;
      tc_fence_after();
      const uint32_t tb = tl + (t & 1) * kBufCols + 8 * eg;
      uint32_t vq[8], vk[8], vv[8];
      tmem_ld8x3(tb + kColGQ, tb + kColGK, tb + kColGV, vq, vk, vv);
      tc_fence_before();
      const int slot = t % kRing, ln = q4 * 32 + lane;
      const int64_t off = ((int64_t)eg * kT + ln) * 8;
      uint4 *pq = reinterpret_cast<uint4 *>(ring_block(a, slot, z, 0, X, Y) + off);
      uint4 *pk = reinterpret_cast<uint4 *>(ring_block(a, slot, z, 1, Y, X) + off);
      uint4 *pv = reinterpret_cast<uint4 *>(ring_block(a, slot, z, 2, Y, X) + off);
      auto pk4 = [](const uint32_t (&v)[8]) {
        return make_uint4(pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1])),
                          pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3])),
                          pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5])),
                          pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7])));
      };
      *pq = pk4(vq);
      *pk = pk4(vk);
      *pv = pk4(vv);
      mbar_arrive(&ctl.drained[t & 1]);
      return true;
    };
    // the row whose gradient blocks still wait in tensor memory (-1: none)
    int pending = -1;
    auto drain_pending = [&](bool block) -> bool {
      if (pending < 0) return true;
      uint64_t *bar = &ctl.gv_done[pending & 1];
      const uint32_t par = (pending >> 1) & 1;
      if (!block && !__any_sync(0xffffffffu, mbar_try_wait(bar, par))) return true;
      if (!wait_bar_warp(bar, par, abort_flag, a.status) || !drain(pending)) return false;
      pending = -1;
      return true;
    };

    bool ok = true;
    for (int t = 0; ok && t < T; ++t) {
      const int b = t & 1, st = t % kStages;
      if (!wait_bar_warp(&ctl.in_full[st], (t / kStages) & 1, abort_flag, a.status) ||
          !wait_bar_warp(&ctl.sdp_full[b], (t >> 1) & 1, abort_flag, a.status) ||
          (t >= 2 &&
           !wait_bar_warp(&ctl.pds_free[b], ((t >> 1) - 1) & 1, abort_flag, a.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint8_t *rb = smem + kOffRow + st * kRowBytes;
      // a per-row key mask: this key drops out of this row
      uint64_t kshift2 = 0ull;
      if (!shared_mask) {
        const uint32_t mw = reinterpret_cast<const uint32_t *>(rb + kLDBytes)[key >> 5];
        if (!((mw >> (key & 31)) & 1u)) kshift2 = f2pack(-INFINITY, -INFINITY);
      }
      uint8_t *dstile = smem + kOffDS + b * kSqBytes;
      const uint32_t sb = tl + b * kBufCols + kColS;
      const uint32_t db = tl + b * kBufCols + kColDP;
#pragma unroll
      for (int c16 = 0; c16 < 2; ++c16) {           // 16 queries at a time
        const int j0 = jbase + 16 * c16;
        // P^T (bf16 pairs) of the 16 queries in pd[0..7], dS^T in pd[8..15]
        uint32_t pd[16];
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {             // 8 queries: one bias chunk
          const int jh = j0 + 8 * h8;
          uint32_t sv[8], dpv[8];
          tmem_ld8x2(sb + jh, db + jh, sv, dpv);
          const int ch = jh >> 3;
          const uint4 bv = *reinterpret_cast<const uint4 *>(brow + ((ch ^ (key & 7)) << 4));
          const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int jj = 2 * e;                    // pair within the 8
            // (-lse*log2e, -lse*log2e, -D, -D) of queries jh+jj, jh+jj+1
            const float4 ld = *reinterpret_cast<const float4 *>(rb + ((jh + jj) >> 1) * 16);
            uint64_t nl2 = f2pack(ld.x, ld.y);
            if (!shared_mask) nl2 = add2(nl2, kshift2);
            const uint64_t bl2 = fma2(f2pack(bf16lo(bw[e]), bf16hi(bw[e])), l2e2, nl2);
            const float2 tt = f2unpack(
                fma2(f2pack(__uint_as_float(sv[jj]), __uint_as_float(sv[jj + 1])), c1x2, bl2));
            const float p0 = ex2_approx(tt.x), p1 = ex2_approx(tt.y);
            const uint64_t ds2 =
                mul2(f2pack(p0, p1), add2(f2pack(__uint_as_float(dpv[jj]),
                                                 __uint_as_float(dpv[jj + 1])),
                                          f2pack(ld.z, ld.w)));
            const int di = (jh - jbase + jj) >> 1;
            db2[di] = add2(db2[di], ds2);
            const float2 ds = f2unpack(ds2);
            pd[4 * h8 + e] = pack_bf16(p0, p1);
            pd[8 + 4 * h8 + e] = pack_bf16(ds.x, ds.y);
          }
        }
        // P^T over this chunk's first 8 S^T columns, dS^T over the next 8 (both
        // halves of the chunk were read above): one 16-column store at the
        // chunk's 16-aligned column
        tmem_st16(sb + j0, pd);
        // dS^T row of this key into the dS tile (the A operand of dQ)
        st_tile_chunk(dstile, key, j0 >> 6, (j0 & 63) >> 3, pd[8], pd[9], pd[10], pd[11]);
        st_tile_chunk(dstile, key, j0 >> 6, ((j0 & 63) >> 3) + 1, pd[12], pd[13], pd[14], pd[15]);
        // the previous row's gradient blocks, if their MMAs are done by now
        if (c16 == 0 && !drain_pending(false)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      tmem_st_wait();
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&ctl.pds_full[b]);
      // the MMA warp issues this row's gradient products now; the previous
      // row's blocks must be out before its dP^T(t + 1) can be computed
      if (!drain_pending(true)) {
        ok = false;
        break;
      }
      pending = t;
    }
    if (ok && T > 0) ok = drain_pending(true);
    // the pair-bias gradient block: summed over every row of the group
    if (ok && y < N) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 v = f2unpack(db2[e]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int x = X * kT + jbase + 2 * e + u;
          const float val = u ? v.y : v.x;
          if (x < N) {
            if (a.ngroups == 1)
              a.dbias[hb + (int64_t)x * a.bX + (int64_t)y * a.bY] = __float2bfloat16_rn(val);
            else
              a.part_db[((int64_t)g * H + h) * N * N + (int64_t)x * N + y] = val;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int bwd_tc_ring_slots() { return kRing; }
int bwd_tc_consumed_flags_per_tile() { return kRing * kReduceWarps; }

bool bwd_tc_plan(int N, int H, int sms, int *nb, int *ngroups, int *gh_per_launch) {
  const int n = (N + kT - 1) / kT;
  *nb = n;
  if (n < 1 || n > kMaxNb || N % 2 != 0) return false;
  const int per_gh = n * n;
  if (per_gh > sms) return false;
  int g = sms / (per_gh * H);
  if (g < 1) g = 1;
  if (g > N) g = N;
  const int rows = (N + g - 1) / g;
  *ngroups = (N + rows - 1) / rows;
  int ghl = sms / per_gh;
  const int total = *ngroups * H;
  if (ghl > total) ghl = total;
  *gh_per_launch = ghl;
  return true;
}

cudaError_t launch_bwd_tc(const BwdMaps &maps, const BwdTcArgs &args, cudaStream_t stream) {
  if (args.N == 0 || args.ghl == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  // Every CTA of a (group, head) pair waits for the others' contributions, so
  // all of them must be resident at once: the planner keeps a launch at no more
  // CTAs than the GPU has SMs, and a CTA takes a whole SM's shared memory, so an
  // otherwise idle GPU runs them all at once. If other work keeps SMs busy for
  // longer than the bounded waits (2 s), the call reports TRI_ATTN_ERR_TIMEOUT
  // in its status word instead of hanging.
  bwd_tc_kernel<<<dim3(args.nb, args.nb, args.ghl), kThreads, kSmemBytes, stream>>>(
      maps.q, maps.k, maps.v, maps.du, args);
  return cudaGetLastError();
}

}  // namespace tri
