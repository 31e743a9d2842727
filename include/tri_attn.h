/*
 * tri_attn.h -- C ABI of the B200 (sm_100a) gated triangle self-attention library.
 *
 * The operation. Triangle attention lets an AlphaFold-family model use a third
 * residue k when it reasons about the pair (i, j); its cost grows cubically
 * with the crop size, and its backward returns gradients for query, key, value
 * and pair bias ("TurboPairFormer accelera fino a 1,73x l'addestramento di
 * OpenFold3 nei test", section "Dove si impiega il tempo"). The gate is fused
 * into the attention op ("HelixFold: An Efficient Implementation of AlphaFold2
 * using PaddlePaddle", proposed methods: fused gated self-attention), and the
 * N^3*H logits are computed tile by tile in on-chip memory and never stored
 * ("MegaFold: Efficient Training of Next-Generation 3D Attention Protein Models
 * on Cross-Platform GPUs", tool 1, EvoFlash-3D). For each attention row r, head
 * h and query x, with c the head dimension:
 *
 *   s_y   = c^-1/2 <q[r,x,h,:], k[r,y,h,:]> + bias[h,x,y] + mu(r,y)
 *   lse   = log sum_y exp(s_y)
 *   out   = sigmoid(gate[r,x,h,:]) * sum_y exp(s_y - lse) v[r,y,h,:]
 *
 * mu(r,y) = 0 if mask[r*mask_row_stride + y] != 0, else -infinity. A row whose
 * keys are all masked yields out = 0 and lse = -infinity and adds nothing to
 * any gradient.
 *
 * Variants. STARTING (around the starting node): row r = i, query x = j, key
 * y = k; pair tensors are read at [r, x] / [r, y] and the bias at [h, x, y].
 * ENDING (around the ending node) runs the same computation on the transposed
 * pair layout: pair tensors are read and written at [x, r] / [y, r], the bias
 * at [h, y, x], and dbias is returned in the bias's own storage layout. The
 * mask and lse are always in the variant's own frame (row, key) / (row, head,
 * query).
 *
 * Layout (all row-major, c fastest, no padding):
 *   q, k, v, gate, out, dout, dq, dk, dv, dgate : [B, N, N, H, c]
 *   bias, dbias                                 : [B, H, N, N]
 *   lse                                         : float32 [B, N, H, N]
 *   mask                                        : uint8 [B, N] (mask_row_stride
 *                                                 0: one key mask per problem,
 *                                                 shared by its rows) or
 *                                                 [B, N, N] (mask_row_stride N);
 *                                                 NULL means every key takes part.
 * B = batch (1 for a single problem, the leading dimension then absent); the B
 * problems are independent. On the tensor-core path they share one launch of
 * each kernel (attention row r of problem b is row b*N + r of the launch); the
 * CUDA-core kernels take them one after another. The row-shard calls take
 * B = 1 only; the on-chip-sum option applies to B = 1 (a batch takes the
 * default backward); B*N is limited like N.
 *
 * Types. dtype BF16: every tensor above except lse and mask is bfloat16. With
 * c == 32 and N % 8 == 0 the contractions run on the tensor cores with fp32
 * accumulation (P and dS rounded to bf16 before their products), softmax and
 * gate arithmetic in fp32; dbias is accumulated in fp32 over all rows and
 * rounded once. Every other bf16 shape runs on the CUDA-core kernels: bf16
 * loads widened to fp32, all arithmetic fp32, each result rounded to bf16
 * once. dtype F32: every tensor is float32 and all arithmetic is fp32 on the
 * CUDA cores (no TF32).
 *
 * Ownership and threading. Every pointer is a caller-owned device pointer,
 * 16-byte aligned, to contiguous memory. The library allocates no device
 * memory and keeps no state between calls: scratch space is the caller's
 * workspace. Outputs are overwritten, never accumulated into. Calls only
 * enqueue work on the given stream and return without synchronising; results
 * are ready once the stream reaches them. Repeated calls on identical inputs
 * give bit-identical outputs (all reductions run in a fixed order, no
 * floating-point atomics). Concurrent calls must use distinct workspaces.
 *
 * Errors. Argument checks happen on the host before anything is enqueued; a
 * call that returns anything but TRI_ATTN_OK has enqueued nothing, except
 * TRI_ATTN_ERR_CUDA, which reports a failed launch. Device-side failures (a
 * bounded wait that ran out) never trap: the kernel records the failure in the
 * workspace status word, fills the affected lse entries with NaN and returns;
 * tri_attn_read_status() reports it.
 */
#ifndef TRI_ATTN_H
#define TRI_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *tri_attn_stream_t;

typedef enum {
    TRI_ATTN_OK = 0,
    TRI_ATTN_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or enum */
    TRI_ATTN_ERR_UNSUPPORTED = 2,  /* valid but not implemented (see limits)    */
    TRI_ATTN_ERR_WORKSPACE = 3,    /* workspace missing or too small            */
    TRI_ATTN_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed         */
    TRI_ATTN_ERR_TIMEOUT = 5,      /* device: a bounded wait ran out            */
    TRI_ATTN_ERR_BOUNDS = 6        /* device: an index check failed             */
} tri_attn_status;

typedef enum { TRI_ATTN_F32 = 0, TRI_ATTN_BF16 = 1 } tri_attn_dtype;
typedef enum { TRI_ATTN_STARTING = 0, TRI_ATTN_ENDING = 1 } tri_attn_variant;

/*
 * Problem description. Limits: N >= 0; H >= 1; 1 <= c <= 64
 * (TRI_ATTN_ERR_UNSUPPORTED above); N * N * H * c < 2^31 * 64. BF16 problems
 * with c == 32 and N % 8 == 0 take the tensor-core kernels (the bias rows are
 * moved by TMA, whose row pitch must be a multiple of 16 bytes); the others,
 * and all F32 problems, the CUDA-core kernels. The rounding-residual option,
 * the on-chip-sum option and row shards need the tensor-core kernels
 * (TRI_ATTN_ERR_UNSUPPORTED, or the default path for the on-chip-sum bit).
 */
typedef struct {
    int64_t N;                /* residues: the pair tensors are N x N           */
    int32_t H;                /* heads                                          */
    int32_t c;                /* head dimension                                 */
    int32_t dtype;            /* tri_attn_dtype                                 */
    int32_t variant;          /* tri_attn_variant                               */
    int64_t mask_row_stride;  /* 0 or N (ignored when mask is NULL)             */
    int32_t batch;            /* independent problems of this size, stacked   */
                              /* along a leading dimension (0 is taken as 1)  */
    int32_t reserved;         /* must be 0                                    */
} tri_attn_problem;

/* Library version, (major << 16) | minor. */
int tri_attn_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *tri_attn_status_string(tri_attn_status status);

/*
 * Description of the CUDA error behind the last call on this host thread that
 * returned TRI_ATTN_ERR_CUDA ("no error" if there was none); a static string
 * owned by the CUDA runtime, never NULL. Host-only, enqueues nothing.
 */
const char *tri_attn_last_cuda_error(void);

/*
 * Workspace the forward needs, in bytes (a status word, plus a transposed copy
 * of the bias for the ENDING variant). Writes *bytes; fails only on an invalid
 * problem.
 */
tri_attn_status tri_attn_fwd_workspace_size(const tri_attn_problem *prob, size_t *bytes);

/*
 * Forward. Reads q, k, v, bias, gate (and mask); writes out and lse. The
 * workspace must hold at least tri_attn_fwd_workspace_size() bytes, 256-byte
 * aligned; its contents on entry do not matter.
 */
tri_attn_status tri_attn_fwd(const tri_attn_problem *prob, const void *q, const void *k,
                             const void *v, const void *bias, const void *gate,
                             const uint8_t *mask, void *out, float *lse, void *workspace,
                             size_t workspace_bytes, tri_attn_stream_t stream);

/* Workspace the backward needs for this problem, in bytes. */
tri_attn_status tri_attn_bwd_workspace_size(const tri_attn_problem *prob, size_t *bytes);

/*
 * Backward of L = sum(dout * out). Reads the forward's inputs and its outputs
 * out and lse (as written by tri_attn_fwd on the same inputs) and dout; writes
 * dq, dk, dv, dgate (pair layout of the inputs) and dbias ([H, N, N], summed
 * over all N attention rows). The probabilities are recomputed from lse once
 * per tile and reused for all four gradients of that tile. Workspace as for
 * the forward, at least tri_attn_bwd_workspace_size() bytes.
 */
tri_attn_status tri_attn_bwd(const tri_attn_problem *prob, const void *q, const void *k,
                             const void *v, const void *bias, const void *gate,
                             const uint8_t *mask, const void *out, const float *lse,
                             const void *dout, void *dq, void *dk, void *dv, void *dbias,
                             void *dgate, void *workspace, size_t workspace_bytes,
                             tri_attn_stream_t stream);

/*
 * Optional per-call settings of the _ex entry points. Zero-initialise, set
 * struct_size = sizeof(tri_attn_launch_opts), then fill what is needed. A
 * struct_size of TRI_ATTN_LAUNCH_OPTS_V1_SIZE (the first four fields) is also
 * accepted; fields past struct_size count as zero.
 *   main_start / main_stop: cudaEvent_t handles (or NULL) that the call
 *   records on its stream immediately before and after its main kernel (the
 *   attention kernel itself, without the small preparation and reduction
 *   kernels), so a caller can time that kernel alone with cudaEventElapsedTime.
 *   out_residual: bf16 path only (NULL on the fp32 path, else
 *   TRI_ATTN_ERR_UNSUPPORTED). Device, caller-owned, 16-byte aligned, shape and
 *   layout of `out` (bf16). The forward writes there the part of each output
 *   element that rounding to bf16 removed, itself rounded to bf16
 *   (bf16(o - bf16(o)) for the fp32 value o); `out` is bit-identical with or
 *   without it. The backward, given the same tensor, forms D = sum_c dout * out
 *   and dgate from out + out_residual instead of the rounded out: the rounding
 *   residual compensation of "TurboPairFormer accelera fino a 1,73x
 *   l'addestramento di OpenFold3 nei test" (section "Accuratezza e
 *   riproducibilita"), which lowers the error of dq, dk and dbias; dv does not
 *   depend on D and is unchanged. NULL: no residual.
 */
typedef struct {
    uint32_t struct_size;
    uint32_t flags;           /* TRI_ATTN_OPT_* bits (backward only), else 0 */
    void *main_start;
    void *main_stop;
    void *out_residual;
} tri_attn_launch_opts;

#define TRI_ATTN_LAUNCH_OPTS_V1_SIZE ((uint32_t)(2 * sizeof(uint32_t) + 2 * sizeof(void *)))

/*
 * flags bit of tri_attn_bwd_ex: sum the per-tile contributions of dq, dk and dv
 * inside the main kernel instead of in a second kernel. The bf16 backward
 * splits every attention row into 128 x 128 query-key tiles, and each row's
 * dq (dk, dv) is a sum over the key (query) tiles of that row ("TurboPairFormer
 * accelera fino a 1,73x l'addestramento di OpenFold3 nei test", section "Dove
 * si impiega il tempo"). By default every tile writes its bf16 contribution to
 * the workspace and a reduction kernel adds them up in tile order. With this
 * bit the tiles of one (row group, head) pair run as co-resident CTAs that pass
 * their contributions through a ring of a few rows in the workspace (resident
 * in L2) to one owner CTA per output tile, which adds them in tile order in
 * fp32 and writes the result: no partial tensors, no reduction kernel, and the
 * results are as deterministic as the default path's (they differ from it only
 * in rounding). Applies when ceil(N / 128) <= 12 and one pair's
 * ceil(N / 128)^2 CTAs fit on the device's SMs; otherwise the call takes the
 * default path. tri_attn_bwd_workspace_size covers both paths. The forward and
 * the fp32 backward reject the bit (TRI_ATTN_ERR_INVALID_ARG).
 */
#define TRI_ATTN_OPT_ONCHIP_SUMS 0x1u

/*
 * flags bit of tri_attn_fwd_ex: compute one key pair in four of the softmax
 * exponentials on the FMA pipe (tri_attn_check_exp2 gives the method and its
 * error bound) instead of the MUFU unit, whose 16 results per clock per SM set
 * the floor of the exponentials of the step. Tensor-core shapes only (the
 * CUDA-core forward ignores it); results differ from the default in the last
 * bits of the affected probabilities. The backward rejects it
 * (TRI_ATTN_ERR_INVALID_ARG).
 */
#define TRI_ATTN_OPT_EXP2_SPLIT 0x2u

/* tri_attn_fwd with options (opts may be NULL: same as tri_attn_fwd). */
tri_attn_status tri_attn_fwd_ex(const tri_attn_problem *prob, const void *q, const void *k,
                                const void *v, const void *bias, const void *gate,
                                const uint8_t *mask, void *out, float *lse, void *workspace,
                                size_t workspace_bytes, tri_attn_stream_t stream,
                                const tri_attn_launch_opts *opts);

/* tri_attn_bwd with options (opts may be NULL: same as tri_attn_bwd). */
tri_attn_status tri_attn_bwd_ex(const tri_attn_problem *prob, const void *q, const void *k,
                                const void *v, const void *bias, const void *gate,
                                const uint8_t *mask, const void *out, const float *lse,
                                const void *dout, void *dq, void *dk, void *dv, void *dbias,
                                void *dgate, void *workspace, size_t workspace_bytes,
                                tri_attn_stream_t stream, const tri_attn_launch_opts *opts);

/*
 * Number of kernel launches one call of the forward (backward = 0), the
 * backward (backward = 1) or the backward with TRI_ATTN_OPT_ONCHIP_SUMS
 * (backward = 2) enqueues for this problem and mask kind (has_mask != 0 for a
 * non-NULL mask), on the current device. Writes *launches; host-only. Any
 * other value of backward: TRI_ATTN_ERR_INVALID_ARG.
 */
tri_attn_status tri_attn_kernel_launches(const tri_attn_problem *prob, int backward,
                                         int has_mask, int32_t *launches);

/*
 * Row shards, for splitting one problem across GPUs (one process per GPU). The
 * attention rows are independent problems that share only the pair bias, whose
 * gradient dbias[h, x, y] sums over every row: the row-wise split of the pair
 * representation across devices ("FastFold: Reducing AlphaFold Training Time
 * from 11 Days to 67 Hours", methods, Dynamic Axial Parallelism) applied to this
 * one operation. A shard is the rows [row_begin, row_begin + row_count) of the
 * variant frame (the first residue index for the starting node, the second for
 * the ending node); row_begin and row_count are multiples of 8 (else
 * TRI_ATTN_ERR_INVALID_ARG); bf16 only (fp32: TRI_ATTN_ERR_UNSUPPORTED).
 * Every pointer is the full [N, N, H, c] / [H, N, N] / [N, H, N] tensor as for
 * tri_attn_fwd / tri_attn_bwd; a shard call reads what its rows need (all keys
 * of its rows, and the whole bias) and writes only its rows of out, lse, dq, dk,
 * dv and dgate. Workspace: the sizes tri_attn_fwd_workspace_size and
 * tri_attn_bwd_workspace_size report. Results on a shard's rows are
 * bit-identical to those of the whole-problem call.
 */
tri_attn_status tri_attn_fwd_rows(const tri_attn_problem *prob, int64_t row_begin,
                                  int64_t row_count, const void *q, const void *k, const void *v,
                                  const void *bias, const void *gate, const uint8_t *mask,
                                  void *out, float *lse, void *workspace, size_t workspace_bytes,
                                  tri_attn_stream_t stream);

/*
 * Backward of a row shard. Instead of dbias it writes dbias_partial (device,
 * caller-owned, fp32, [H, N, N] in the layout of dbias): the sum over the
 * shard's rows, in a fixed order. The full dbias is the sum of every shard's
 * partial; tri_attn_dbias_reduce adds gathered partials in rank order and rounds
 * to bf16 once, so every rank obtains the same bits.
 */
tri_attn_status tri_attn_bwd_rows(const tri_attn_problem *prob, int64_t row_begin,
                                  int64_t row_count, const void *q, const void *k, const void *v,
                                  const void *bias, const void *gate, const uint8_t *mask,
                                  const void *out, const float *lse, const void *dout, void *dq,
                                  void *dk, void *dv, float *dbias_partial, void *dgate,
                                  void *workspace, size_t workspace_bytes,
                                  tri_attn_stream_t stream);

/*
 * dbias (bf16, [H, N, N]) = sum over i = 0 .. count-1, in that order, of the fp32
 * partials[i] ([count][H][N][N], contiguous, 16-byte aligned; the all-gathered
 * outputs of tri_attn_bwd_rows in rank order), rounded once. One kernel,
 * asynchronous on `stream`. TRI_ATTN_ERR_INVALID_ARG for count < 1, a bad N or
 * H, or NULL / misaligned pointers.
 */
tri_attn_status tri_attn_dbias_reduce(const float *partials, int32_t count, int64_t N, int32_t H,
                                      void *dbias, tri_attn_stream_t stream);

/* Size of the fixed scratch area behind tri_attn_fwd_noalloc, per GPU. */
#define TRI_ATTN_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/*
 * Forward that allocates nothing and takes no workspace. The pages describe no
 * such entry point; it exists for callers that are not allowed to allocate
 * device memory themselves: code inside a framework or inference engine whose
 * allocator owns every device byte and hands out none for foreign scratch, and
 * latency-critical loops that cannot afford the implicit device-wide
 * synchronisation of cudaMalloc/cudaFree. Arguments, layout and results are
 * those of tri_attn_fwd without the workspace.
 *
 * Scratch: a device array of TRI_ATTN_NOALLOC_SCRATCH_BYTES compiled into the
 * library. Every GPU on which the library is used holds that array until the
 * process exits. A problem whose tri_attn_fwd_workspace_size() exceeds it is
 * rejected with TRI_ATTN_ERR_WORKSPACE before anything is enqueued (starting
 * node: any size up to the N limit; ending node: B*H*N*N*2 bytes must also fit).
 *
 * The first call in a CUDA context looks up the array's device address with
 * that context's device current and keeps it, keyed by the context's unique
 * id; a later call in another context (a new primary context after
 * cudaDeviceReset, or one the caller made current) looks it up again. Make the
 * first call of each context before any stream capture. The call itself never
 * calls cudaMalloc, cudaFree or any allocating routine.
 *
 * All calls share the one array and leave their scratch in it; every call
 * rewrites what it reads. Calls whose work overlaps on the GPU (other streams,
 * other host threads) race on the array and corrupt each other's results:
 * serialise them. The status word lives inside the private array, so
 * tri_attn_read_status() cannot reach it: for this entry point NaN in lse is
 * the only sign of a device-side failure (a bounded wait that ran out).
 */
tri_attn_status tri_attn_fwd_noalloc(const tri_attn_problem *prob, const void *q, const void *k,
                                     const void *v, const void *bias, const void *gate,
                                     const uint8_t *mask, void *out, float *lse,
                                     tri_attn_stream_t stream);

/*
 * Device status word of the last call that used this workspace: synchronises
 * the stream, copies the word to the host and stores a tri_attn_status in
 * *device_status. Returns TRI_ATTN_ERR_CUDA if the copy itself fails.
 */
tri_attn_status tri_attn_read_status(const void *workspace, int32_t *device_status,
                                     tri_attn_stream_t stream);

/*
 * The same device status word returned as the call's own status: synchronises
 * the stream and returns what the last call that used this workspace recorded
 * on the device (TRI_ATTN_OK, TRI_ATTN_ERR_TIMEOUT for a bounded wait that ran
 * out, TRI_ATTN_ERR_BOUNDS for a tile the kernel refused). Returns
 * TRI_ATTN_ERR_INVALID_ARG for a NULL workspace and TRI_ATTN_ERR_CUDA if the
 * synchronisation or the copy fails. The workspace is caller-owned device
 * memory laid out by tri_attn_fwd / tri_attn_bwd (the word sits at offset 0).
 * The pages define no status channel; this is the boundary's query call.
 */
tri_attn_status tri_attn_get_status(const void *workspace, tri_attn_stream_t stream);

/*
 * Diagnostic of the failure path (no counterpart on the pages): enqueues one
 * small kernel whose warp waits on a barrier that nothing ever completes,
 * using the same bounded wait (about 2 s) as the forward and backward kernels.
 * The wait gives up and the kernel writes TRI_ATTN_ERR_TIMEOUT to the status
 * word at the start of `workspace` (which it first resets); it never traps or
 * faults, so the stream and context stay usable. Read the result with
 * tri_attn_read_status(). workspace: device, 16-byte aligned, at least 256
 * bytes, caller-owned. Returns TRI_ATTN_ERR_WORKSPACE for a missing, misaligned
 * or short workspace, TRI_ATTN_ERR_CUDA if the launch fails.
 */
tri_attn_status tri_attn_check_wait_timeout(void *workspace, size_t workspace_bytes,
                                            tri_attn_stream_t stream);

/*
 * Diagnostic of the forward's two exp2 evaluations (no counterpart on the
 * pages): for each of the n fp32 exponents x (device), y_fma receives the
 * FMA-pipe polynomial evaluation that TRI_ATTN_OPT_EXP2_SPLIT uses (Cody-Waite
 * reduction, degree-4 minimax polynomial, relative error below 2.7e-6 for
 * -125 <= x <= 126, inputs below -125 treated as -125) and y_mufu the hardware
 * approximation (ex2.approx.ftz). Device buffers of n floats, caller-owned; one
 * kernel on `stream`. TRI_ATTN_ERR_INVALID_ARG for n < 0 or NULL pointers.
 */
tri_attn_status tri_attn_check_exp2(const float *x, float *y_fma, float *y_mufu, int64_t n,
                                    tri_attn_stream_t stream);

/*
 * Diagnostic of the tensor-core instruction the kernels are built from (no
 * counterpart on the pages): tcgen05.mma kind::f16, bf16 operands, fp32
 * accumulator in tensor memory, M = 128 and K = 16 per instruction, N = n in
 * {32, 64, 128, 256}. Each of `ctas` CTAs (1 .. 1024; one per SM when ctas is
 * the SM count) issues `instructions` (1 .. 2^24, rounded up to a multiple of 8)
 * instructions back to back
 * into one accumulator and writes the SM clock cycles from the first issue to
 * their completion to cycles[cta] (device, caller-owned, `ctas` entries).
 * layout 0: both operands K-major with the 64-byte swizzle (the S = Q K^T form);
 * layout 1: both MN-major (the dV = P^T dU form); layout 2: A read from tensor
 * memory, B MN-major (the O += P V form); layouts 1 and 2 take n = 32. The
 * shared-memory operands are zeros; the tensor-memory one is whatever the
 * columns hold (the timing does not depend on the values). *status (device int32) is set to 0, or to
 * TRI_ATTN_ERR_TIMEOUT if the completion did not come within the bounded wait.
 * TRI_ATTN_ERR_INVALID_ARG for other n, layout or counts, or NULL pointers.
 */
tri_attn_status tri_attn_probe_mma(int32_t n, int32_t layout, int32_t ctas, int32_t instructions,
                                   unsigned long long *cycles, int32_t *status,
                                   tri_attn_stream_t stream);

/* ------------------------------------------------ triangle multiplication --
 *
 * The contraction at the core of the triangle multiplicative update, the other
 * pair operation the pages' kernels accelerate ("TurboPairFormer accelera fino
 * a 1,73x l'addestramento di OpenFold3 nei test", section "Dove si impiega il
 * tempo"; the pages print no formula, this is the standard AlphaFold-family
 * one). Per channel c, on channel-major bf16 stacks x[c][r][s] at
 * (c*N + r)*N + s:
 *   TRI_MUL_OUTGOING: t[c][i][j] = sum_k a[c][i][k] * b[c][j][k]
 *   TRI_MUL_INCOMING: t[c][i][j] = sum_k a[c][k][i] * b[c][k][j]
 * fp32 accumulation on the tensor cores, bf16 results. The backward of
 * L = sum(dt * t) gives da and db in the layout of a and b:
 *   outgoing: da[c][i][k] = sum_j dt[c][i][j] b[c][j][k],
 *             db[c][j][k] = sum_i dt[c][i][j] a[c][i][k]
 *   incoming: da[c][k][i] = sum_j dt[c][i][j] b[c][k][j],
 *             db[c][k][j] = sum_i dt[c][i][j] a[c][k][i]
 * Pointers: device, caller-owned, 16-byte aligned, contiguous [C][N][N] bf16.
 * N must be a multiple of 8 (TRI_ATTN_ERR_UNSUPPORTED otherwise); N = 0
 * returns TRI_ATTN_OK after the argument checks and enqueues nothing. The workspace (device, 16-byte aligned, tri_mul_workspace_size bytes)
 * holds the status word that tri_attn_read_status() reads. Calls are
 * asynchronous on the stream, allocate nothing and are deterministic (each
 * output element is one fixed-order tensor-core accumulation).
 */
typedef enum { TRI_MUL_OUTGOING = 0, TRI_MUL_INCOMING = 1 } tri_mul_direction;

typedef struct {
    int64_t N;          /* residues */
    int32_t C;          /* channels (independent N x N products) */
    int32_t direction;  /* tri_mul_direction */
} tri_mul_problem;

tri_attn_status tri_mul_workspace_size(const tri_mul_problem *prob, size_t *bytes);

tri_attn_status tri_mul_fwd(const tri_mul_problem *prob, const void *a, const void *b, void *t,
                            void *workspace, size_t workspace_bytes, tri_attn_stream_t stream);

tri_attn_status tri_mul_bwd(const tri_mul_problem *prob, const void *a, const void *b,
                            const void *dt, void *da, void *db, void *workspace,
                            size_t workspace_bytes, tri_attn_stream_t stream);

/*
 * The full triangle multiplicative update around the contraction, forward and
 * backward ("TurboPairFormer accelera fino a 1,73x l'addestramento di OpenFold3
 * nei test", sections "Dove si impiega il tempo" and "Benchmark di
 * addestramento", name it beside triangle attention; the pages print no
 * formula, the standard AlphaFold-family form is taken). Per pair position of
 * z [N][N][cz] (bf16):
 *   x = LayerNorm(z)                                   (over cz, biased variance)
 *   [ap | ag | bp | bg | gl] = x W_in + b_in           W_in [cz][4c + cz]
 *   a = sigmoid(ag) ap,  b = sigmoid(bg) bp            [N][N][c]
 *   t = the outgoing or incoming contraction of a and b (tri_mul_fwd)
 *   y = sigmoid(gl) (LayerNorm_out(t) W_o + b_o)       W_o [c][cz], y [N][N][cz] bf16
 * Limits: cz and c in {64, 128, 192, 256}, N a multiple of 8
 * (TRI_ATTN_ERR_UNSUPPORTED otherwise), eps > 0.
 */
typedef struct {
    int64_t N;          /* residues */
    int32_t cz;         /* channels of z and y */
    int32_t c;          /* channels of a, b and t */
    int32_t direction;  /* tri_mul_direction */
    float eps;          /* epsilon of both LayerNorms */
} tri_mul_update_problem;

/* Parameters (device, caller-owned, 16-byte aligned). */
typedef struct {
    const float *ln_gamma, *ln_beta;          /* fp32 [cz] */
    const void *w_in;                          /* bf16 [cz][4c + cz]: W_ap W_ag W_bp W_bg W_g */
    const float *b_in;                         /* fp32 [4c + cz] */
    const float *ln_out_gamma, *ln_out_beta;   /* fp32 [c] */
    const void *w_o;                           /* bf16 [c][cz] */
    const float *b_o;                          /* fp32 [cz] */
} tri_mul_update_params;

/* Parameter gradients (device, fp32, the shapes of the parameters). */
typedef struct {
    float *ln_gamma, *ln_beta, *w_in, *b_in, *ln_out_gamma, *ln_out_beta, *w_o, *b_o;
} tri_mul_update_grads;

/*
 * Bytes of the activations the forward keeps for the backward (`saved`) and of
 * the scratch either call needs (`workspace`, the larger of the two calls').
 */
tri_attn_status tri_mul_update_sizes(const tri_mul_update_problem *prob, size_t *saved_bytes,
                                     size_t *workspace_bytes);

/*
 * Forward: reads z, writes y and the saved activations (caller-owned, at least
 * saved_bytes, kept unchanged until the backward has run). Returns before the
 * work completes; the workspace's first word is the status word
 * (tri_attn_get_status).
 */
tri_attn_status tri_mul_update_fwd(const tri_mul_update_problem *prob,
                                   const tri_mul_update_params *params, const void *z, void *y,
                                   void *saved, size_t saved_bytes, void *workspace,
                                   size_t workspace_bytes, tri_attn_stream_t stream);

/*
 * Backward of L = sum(dy * y): dz (bf16, shape of z) and every parameter
 * gradient (overwritten, fp32, summed over the pair positions in a fixed
 * order). `saved` is what the forward of the same z and parameters wrote.
 */
tri_attn_status tri_mul_update_bwd(const tri_mul_update_problem *prob,
                                   const tri_mul_update_params *params, const void *z,
                                   const void *saved, size_t saved_bytes, const void *dy,
                                   void *dz, const tri_mul_update_grads *grads, void *workspace,
                                   size_t workspace_bytes, tri_attn_stream_t stream);

/* ------------------------------------------ LayerNorm and projections --
 *
 * The steps either side of the attention. The pages put LayerNorm at 14% of
 * AlphaFold training time, at 10% of its theoretical speed before optimisation
 * ("알파폴드 초기 학습 시간을 10시간으로 단축하는 ScaleFold", Stats), and fuse
 * the gated self-attention with the projections around it ("HelixFold: An
 * Efficient Implementation of AlphaFold2 using PaddlePaddle", proposed methods);
 * they print neither, and this is the standard AlphaFold-family block. Per pair
 * position (a row of z, cz channels; rows = N*N per batch element):
 *
 *   input side   x       = (z - mean) / sqrt(var + eps) * gamma + beta
 *                          (biased variance over the cz channels)
 *                q|k|v|g = x w_qkvg (+ b_g on g only)   -> [rows][H*c] each
 *                bias[h] = x w_b[:, h]                  -> [batch][H][rows]
 *   output side  y       = o w_o + b_o                  -> [rows][cz]
 *
 * q, k, v, g and bias are laid out exactly as tri_attn_fwd takes them (g are
 * the gate logits; [rows][H*c] is [N, N, H, c]); o is the attention's output.
 * The backward entry points return the gradient of L = sum(dq q) + sum(dk k) +
 * sum(dv v) + sum(dg g) + sum(dbias bias), or L = sum(dy y).
 *
 * Types: z, x, q, k, v, g, bias, o, y and every activation gradient are bf16;
 * w_qkvg, w_b, w_o are bf16; gamma, beta, b_g, b_o, stats and every parameter
 * gradient are float32. LayerNorm statistics and the row sums are fp32; the
 * products run on the tensor cores with fp32 accumulation. x is rounded to bf16
 * once and both the projections and the bias read that rounded x.
 *
 * Layouts (row-major, no padding): z, x, y, dz, dy [batch*rows][cz];
 * q, k, v, g and their gradients, o, do [batch*rows][H*c]; bias, dbias
 * [batch][H][rows]; stats [batch*rows][2] = (mean, 1/sqrt(var + eps));
 * w_qkvg [cz][4*H*c] (the q, k, v, g blocks side by side); b_g [H*c];
 * w_b [cz][H]; w_o [H*c][cz]; gamma, beta, b_o [cz]. Parameter gradients have
 * their parameter's shape.
 *
 * Limits (TRI_ATTN_ERR_UNSUPPORTED otherwise): cz in {64, 128, 192, 256};
 * 1 <= H <= 8; H*c in {64, 128, 192, 256}; batch*rows < 2^31. rows = 0 or batch = 0
 * computes nothing but still zeroes the parameter gradients; the activation
 * pointers may then be NULL (those of the parameters and their gradients may not).
 *
 * Ownership, errors, determinism: as for the attention. Every pointer is a
 * caller-owned, 16-byte aligned device pointer (x and stats too: the forward
 * writes them, the backward reads them). The workspace (tri_proj_workspace_size
 * bytes, one size for all four calls, device, 16-byte aligned) holds the status
 * word that tri_attn_read_status() reads, the input backward's dx in fp32
 * ([batch*rows][cz]) and the fp32 partial sums; parameter gradients are summed
 * over the rows in a fixed order (per-block or per-split partials, then one
 * ordered sum), so repeated calls are bit-identical. Device-side bounded waits
 * that run out set TRI_ATTN_ERR_TIMEOUT in the status word; nothing traps.
 */
typedef struct {
    int64_t rows;   /* pair positions per batch element (N*N) */
    int32_t batch;  /* independent pair maps, >= 0 */
    int32_t cz;     /* channels of z */
    int32_t H;      /* heads */
    int32_t c;      /* channels per head */
    float eps;      /* LayerNorm epsilon (> 0) */
    int32_t reserved; /* must be 0 */
} tri_proj_problem;

tri_attn_status tri_proj_workspace_size(const tri_proj_problem *prob, size_t *bytes);

/* x, stats, q, k, v, g, bias from z. */
tri_attn_status tri_proj_in_fwd(const tri_proj_problem *prob, const void *z, const float *gamma,
                                const float *beta, const void *w_qkvg, const float *b_g,
                                const void *w_b, void *x, float *stats, void *q, void *k,
                                void *v, void *g, void *bias, void *workspace,
                                size_t workspace_bytes, tri_attn_stream_t stream);

/* dz and the parameter gradients from dq, dk, dv, dg, dbias (x and stats as
 * the forward wrote them). */
tri_attn_status tri_proj_in_bwd(const tri_proj_problem *prob, const void *z, const float *gamma,
                                const void *w_qkvg, const void *w_b, const void *x,
                                const float *stats, const void *dq, const void *dk,
                                const void *dv, const void *dg, const void *dbias, void *dz,
                                float *dgamma, float *dbeta, float *dw_qkvg, float *db_g,
                                float *dw_b, void *workspace, size_t workspace_bytes,
                                tri_attn_stream_t stream);

/* y = o w_o + b_o. */
tri_attn_status tri_proj_out_fwd(const tri_proj_problem *prob, const void *o, const void *w_o,
                                 const float *b_o, void *y, void *workspace,
                                 size_t workspace_bytes, tri_attn_stream_t stream);

/* do, dw_o, db_o from dy. */
tri_attn_status tri_proj_out_bwd(const tri_proj_problem *prob, const void *o, const void *w_o,
                                 const void *dy, void *do_, float *dw_o, float *db_o,
                                 void *workspace, size_t workspace_bytes,
                                 tri_attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TRI_ATTN_H */
