// Launch interfaces of the bf16 tcgen05 kernels (forward, backward) and of
// the small preparation kernels they share.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace tri {

// ------------------------------------------------------------------ forward --
// Pair-tensor maps list their dimensions by increasing stride: (c, h, x, r, b)
// when the query index has the smaller stride (x_inner = 1, starting node),
// else (c, h, r, x, b), b the problem of a batch; the box is 32 channels x 1
// head x 128 queries x 1 row x 1 problem, so a tile lands in shared memory as
// 128 rows of 64 bytes (64-byte swizzle). The bias map is (y, x, b*H + h) in
// the variant frame, box (64, 128, 1), 128-byte swizzle. Attention rows of the
// batch count on across problems: row b*N + r is row r of problem b.
struct FwdMaps {
  CUtensorMap q, k, v;
  CUtensorMap bias;
};

struct FwdArgs {
  int N, H;
  int row0, row_end;                 // attention rows of this launch (multiples of 8)
  int exp2_split;                    // host-side: one key pair in four takes the FMA-pipe exp2
  int x_inner;                       // dimension order of the pair maps (see above)
  float scale;                       // c^-1/2
  int64_t sR, sX;                    // pair strides of the variant frame (elements)
  const __nv_bfloat16 *gate;
  __nv_bfloat16 *out;
  __nv_bfloat16 *out_res;            // rounding residual of out (bf16) or null
  float *lse;
  const uint32_t *mask_bits;         // [rows][ceil(N/128)*4] key bits, 0 beyond N
  int64_t mask_bits_stride;          // words per row of bits
  int mask_per_row;                  // 1: a row of bits per attention row, 0: one per problem
  int32_t *status;
};

int fwd_bf16_rows_per_cta();
int fwd_bf16_key_tile();           // keys per K/V tile (rows of the K and V boxes)
cudaError_t launch_fwd_bf16(const FwdMaps &maps, const FwdArgs &args, cudaStream_t stream);

// ----------------------------------------------------------------- backward --
struct BwdMaps {
  CUtensorMap q, k, v;   // as for the forward
  CUtensorMap du;        // dU = dout * sigmoid(g), compact variant frame, dims (c, h, x, r)
  CUtensorMap bias;
};

struct BwdArgs {
  int N, H, B;                       // B problems of N x N pairs and H heads
  int row0, row_end;                 // attention rows of this launch (of the batch)
  int x_inner;
  int nb;                            // tiles per axis, ceil(N / 128)
  float scale;
  int64_t sR, sX;                    // pair strides of the variant frame (outputs)
  const float *lse;                  // [B*N, H, N] natural log
  const float *D;                    // [B*N, H, N] sum_c dout * out
  const uint32_t *mask_bits;
  int64_t mask_bits_stride;          // words per row of bits
  int mask_per_row;                  // 1: a row of bits per attention row, 0: one per problem
  // bf16 tile contributions, [tile][B*N rows][H][2][N][16] (16-channel halves):
  // part_q over key tiles yb, part_k and part_v over query tiles xb
  __nv_bfloat16 *part_q, *part_k, *part_v;
  float *part_db;                    // [ngroups][B*H, N, N] variant frame (used when dbias is null)
  __nv_bfloat16 *dbias;              // final dbias (one row group covering every row), else null
  int64_t bX, bY;                    // dbias strides of the variant frame
  int ngroups, rows_per_group;
  int32_t *status;
};

// Tiling of the backward over `rows` attention rows: tiles per axis and row groups
// (never more than bwd_bf16_max_groups(N, H)).
void bwd_bf16_plan(int N, int H, int rows, int *nxb, int *ngroups);
int bwd_bf16_max_groups(int N, int H);
cudaError_t launch_bwd_bf16(const BwdMaps &maps, const BwdArgs &args, cudaStream_t stream);

// ------------------------------------------- backward with on-chip sums --
// The backward whose cross-tile sums of dq, dk and dv run inside the kernel
// (bwd_tc.cu). One CTA per (query tile X, key tile Y, local group-head pair z);
// the CTAs of one pair exchange their gradient blocks through `ring` and the
// integer flags, so all CTAs of a launch must be resident at once.
struct BwdTcArgs {
  int N, H;
  int x_inner;
  int nb;                            // tiles per axis, ceil(N / 128) (at most 12)
  int ngroups, rows_per_group;       // attention rows split into groups
  int gh0, ghl;                      // first (group, head) pair of this launch, pairs in it
  float scale;
  int64_t sR, sX;                    // pair strides of the variant frame (outputs)
  int64_t bX, bY;                    // bias and dbias strides of the variant frame
  const __nv_bfloat16 *bias;         // the caller's bias (variant frame through bX, bY)
  const float4 *LD;                  // [N][H][N/2]: (-lse*log2e) and (-D) of query pairs
  const uint32_t *mask_bits;
  int64_t mask_bits_stride;
  __nv_bfloat16 *dq, *dk, *dv;       // results (variant frame strides)
  __nv_bfloat16 *dbias;              // ngroups == 1
  float *part_db;                    // [ngroups][H, N, N] (ngroups > 1)
  __nv_bfloat16 *ring;               // [slots][ghl][3][nb][nb][4][128][8] gradient blocks
  int32_t *exported;                 // [ngroups*H][nb][nb] rows exported per CTA
  int32_t *consumed_q, *consumed_kv; // [ngroups*H][nb][slots][2] rows summed, per owner warp
  int32_t *status;
};

int bwd_tc_ring_slots();
// Consumed flags per output tile (ring slots x owner warps).
int bwd_tc_consumed_flags_per_tile();
// Tiling of the on-chip-sum backward for `sms` SMs; false when it does not
// apply (more than 12 tiles per axis, odd N, or more CTAs per pair than SMs).
bool bwd_tc_plan(int N, int H, int sms, int *nb, int *ngroups, int *gh_per_launch);
cudaError_t launch_bwd_tc(const BwdMaps &maps, const BwdTcArgs &args, cudaStream_t stream);

// ------------------------------------------------------------ preparation --
// Packs the key mask of every attention row into bits (0 beyond N), resets the
// status word and zeroes `nzero` int32 words at `zero` (counters; may be 0).
// rows = N for a per-row mask, 1 for a shared one.
cudaError_t launch_mask_bits(const Frame &f, uint32_t *bits, int64_t rows, int64_t words_per_row,
                             int32_t *status, int32_t *zero, int64_t nzero, cudaStream_t stream);
// biasT[h][x][y] = bias[h][y][x] (bf16), for the ending-node variant.
cudaError_t launch_bias_transpose(const __nv_bfloat16 *bias, __nv_bfloat16 *biasT, int N, int H,
                                  cudaStream_t stream);
// dq, dk, dv (variant frame strides) = scale_q/k/v * the sum over nb tiles of
// the bf16 contributions [tile][row][H][2][N][16], added in tile order.
cudaError_t launch_partial_reduce_bf16(const Frame &f, const __nv_bfloat16 *part_q,
                                       const __nv_bfloat16 *part_k, const __nv_bfloat16 *part_v,
                                       int nb, float scale, __nv_bfloat16 *dq, __nv_bfloat16 *dk,
                                       __nv_bfloat16 *dv, cudaStream_t stream);
// du (compact variant frame, bf16) = dout * sigmoid(g); D = sum_c dout * out;
// dgate (storage layout) = dout * out * (1 - sigmoid(g)); out + out_res in
// place of out when out_res (the forward's rounding residual) is given.
// With lse and LD given (the on-chip-sum backward), D goes into LD instead:
// LD[(r*H + h)*(N/2) + x/2] = (-lse*log2e of x, x+1; -D of x, x+1), with an
// exponent of -inf for a query whose lse is -inf (all keys masked).
cudaError_t launch_bwd_pre_bf16(const Frame &f, const __nv_bfloat16 *gate,
                                const __nv_bfloat16 *out, const __nv_bfloat16 *out_res,
                                const __nv_bfloat16 *dout,
                                __nv_bfloat16 *du, float *D, __nv_bfloat16 *dgate,
                                const float *lse, float *LD, cudaStream_t stream);

}  // namespace tri
