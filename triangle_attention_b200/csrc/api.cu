// C ABI of the library (declared in include/tri_attn.h): argument checks,
// workspace carving, TMA tensor-map encoding and dispatch to the kernels.
// Nothing here allocates device memory or keeps state between calls.
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <type_traits>
#include <utility>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/tri_attn.h"
#include "bf16.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "mul_update.cuh"
#include "proj.cuh"

namespace {

using tri::Frame;

constexpr size_t kAlign = 256;
constexpr int64_t kMaxN = 1 << 16;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tri_attn_status check_problem(const tri_attn_problem *p) {
  if (!p) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->N < 0 || p->N > kMaxN || p->H < 1 || p->H > 4096 || p->c < 1)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (p->dtype != TRI_ATTN_F32 && p->dtype != TRI_ATTN_BF16) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->variant != TRI_ATTN_STARTING && p->variant != TRI_ATTN_ENDING)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (p->mask_row_stride != 0 && p->mask_row_stride != p->N) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->batch < 0 || p->reserved != 0 || (int64_t)std::max(p->batch, 1) * p->N > kMaxN)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (p->c > 64) return TRI_ATTN_ERR_UNSUPPORTED;
  return TRI_ATTN_OK;
}

// Problems in the batch (0 is taken as 1).
int64_t batch_of(const tri_attn_problem *p) { return p->batch > 1 ? p->batch : 1; }

// bf16 problems the tensor-core kernels take (head dimension 32, N a multiple of
// 8); every other problem runs on the CUDA-core kernels.
bool tc_shape(const tri_attn_problem *p) {
  // (the backward grid's third dimension counts heads x row groups x problems)
  return p->dtype == TRI_ATTN_BF16 && p->c == 32 && p->N % 8 == 0 &&
         (int64_t)p->H * batch_of(p) * tri::bwd_bf16_max_groups((int)p->N, p->H) <= 65535;
}

Frame make_frame(const tri_attn_problem *p, const uint8_t *mask, int32_t *status) {
  Frame f;
  f.N = (int)p->N;
  f.H = p->H;
  f.c = p->c;
  f.variant = p->variant;
  const int64_t N = p->N, H = p->H, C = p->c;
  if (p->variant == TRI_ATTN_STARTING) {
    f.sR = N * H * C;
    f.sX = H * C;
    f.bX = N;
    f.bY = 1;
  } else {
    f.sR = H * C;
    f.sX = N * H * C;
    f.bX = 1;
    f.bY = N;
  }
  f.mask = mask;
  f.mask_stride = mask ? p->mask_row_stride : 0;
  f.status = status;
  f.B = (int)batch_of(p);
  f.row0 = 0;
  f.row_end = (int)(p->N * f.B);     // attention rows of every problem of the batch, in order
  return f;
}


// ------------------------------------------------------- workspace layout --

struct Carver {
  char *base;
  size_t off = 0;
  explicit Carver(void *b) : base(static_cast<char *>(b)) {}
  void *take(size_t bytes) {
    void *p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  }
};

// Offsets between consecutive problems of a batch: the pair and bias tensors in
// bytes (their element type varies), lse in floats, the mask in bytes.
struct ProblemStrides {
  int64_t pair, bias, lse, mask;
};
ProblemStrides problem_strides(const tri_attn_problem *p, bool has_mask) {
  const int64_t N = p->N;
  const int64_t es = p->dtype == TRI_ATTN_F32 ? 4 : 2;
  return {N * N * p->H * p->c * es, (int64_t)p->H * N * N * es, N * p->H * N,
          has_mask ? (p->mask_row_stride == N ? N * N : N) : 0};
}
// `base` advanced by `bytes`.
template <typename T> T *at(T *base, int64_t bytes) {
  return reinterpret_cast<T *>(reinterpret_cast<
      typename std::conditional<std::is_const<T>::value, const char, char>::type *>(base) +
                               bytes);
}

// Rows of packed key bits: one per attention row of every problem (a per-row
// mask), else one per problem.
int64_t mask_rows(const tri_attn_problem *p, bool has_mask) {
  return (has_mask && p->mask_row_stride == p->N) ? p->N * batch_of(p) : batch_of(p);
}

int64_t mask_words_per_row(const tri_attn_problem *p) { return ((p->N + 127) / 128) * 4; }

struct FwdWs {
  int32_t *status;
  uint32_t *mask_bits;
  __nv_bfloat16 *biasT;
};

// Worst case over the mask argument (a per-row mask needs N rows of bits).
size_t carve_fwd(const tri_attn_problem *p, void *ws, bool per_row_mask, FwdWs *out) {
  Carver c(ws);
  FwdWs w{};
  w.status = static_cast<int32_t *>(c.take(sizeof(int32_t)));
  if (tc_shape(p)) {
    const int64_t rows = (per_row_mask ? p->N : 1) * batch_of(p);
    w.mask_bits = static_cast<uint32_t *>(c.take(sizeof(uint32_t) * rows * mask_words_per_row(p)));
    if (p->variant == TRI_ATTN_ENDING)
      w.biasT = static_cast<__nv_bfloat16 *>(
          c.take(2 * (size_t)p->H * p->N * p->N * batch_of(p)));
  }
  if (out) *out = w;
  return c.off;
}

// SMs of the current device (the B200's 148 when no device answers, as on a
// build host): the on-chip-sum backward sizes its grid, and so its workspace, by it.
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

struct BwdWs {
  FwdWs fw;
  void *du;
  float *D;
  // fp32 path: partial sums per tile, reduced by a second kernel
  float *part_dq, *part_dk, *part_dv;
  // bf16 path without on-chip sums: bf16 contributions per tile, reduced by a
  // second kernel
  __nv_bfloat16 *bpart_q, *bpart_k, *bpart_v;
  float *part_db;
  int ntile, ngroups;
  // bf16 path with on-chip sums (tc): lse/D pairs, exchange ring and flags
  bool tc;
  int ghl;                      // (group, head) pairs per launch
  float *LD;
  __nv_bfloat16 *ring;
  int32_t *flags;               // exported | consumed_q | consumed_kv
  int64_t nflags;
};

size_t carve_bwd(const tri_attn_problem *p, void *ws, bool per_row_mask, bool onchip,
                 BwdWs *out) {
  Carver c(ws);
  BwdWs w{};
  w.fw.status = static_cast<int32_t *>(c.take(sizeof(int32_t)));
  const size_t pair = (size_t)p->N * p->N * p->H * p->c;
  const size_t nn = (size_t)p->N * p->N;
  const size_t B = (size_t)batch_of(p);
  if (tc_shape(p)) {
    const int64_t rows = (per_row_mask ? p->N : 1) * (int64_t)B;
    w.fw.mask_bits =
        static_cast<uint32_t *>(c.take(sizeof(uint32_t) * rows * mask_words_per_row(p)));
    w.tc = onchip && B == 1 &&
           tri::bwd_tc_plan((int)p->N, p->H, sm_count(), &w.ntile, &w.ngroups, &w.ghl);
    if (w.tc) {
      const int64_t gh = (int64_t)w.ngroups * p->H, nb = w.ntile;
      w.du = c.take(2 * pair);
      w.LD = static_cast<float *>(c.take(8 * nn * p->H));
      w.ring = static_cast<__nv_bfloat16 *>(
          c.take((size_t)tri::bwd_tc_ring_slots() * w.ghl * 3 * nb * nb * 128 * 32 * 2));
      w.nflags = gh * nb * nb + 2 * gh * nb * tri::bwd_tc_consumed_flags_per_tile();
      w.flags = static_cast<int32_t *>(c.take(4 * (size_t)w.nflags));
    } else {
      if (p->variant == TRI_ATTN_ENDING)
        w.fw.biasT = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)p->H * nn * B));
      // planned per problem, so that a problem of a batch is summed in the same
      // order as the same problem alone
      tri::bwd_bf16_plan((int)p->N, p->H, (int)p->N, &w.ntile, &w.ngroups);
      w.du = c.take(2 * pair * B);
      w.D = static_cast<float *>(c.take(4 * nn * p->H * B));
      w.bpart_q = static_cast<__nv_bfloat16 *>(c.take(2 * pair * B * (size_t)w.ntile));
      w.bpart_k = static_cast<__nv_bfloat16 *>(c.take(2 * pair * B * (size_t)w.ntile));
      w.bpart_v = static_cast<__nv_bfloat16 *>(c.take(2 * pair * B * (size_t)w.ntile));
    }
  } else {
    tri::f32_bwd_plan(make_frame(p, nullptr, nullptr), &w.ntile, &w.ngroups);
    w.du = c.take(4 * pair);
    w.D = static_cast<float *>(c.take(4 * nn * p->H));
    w.part_dq = static_cast<float *>(c.take(4 * pair * (size_t)w.ntile));
    w.part_dk = static_cast<float *>(c.take(4 * pair * (size_t)w.ntile));
    w.part_dv = static_cast<float *>(c.take(4 * pair * (size_t)w.ntile));
  }
  if (tc_shape(p) && !w.tc) {
    // per-group dbias sums: also taken by a row-shard call, whose groups split
    // fewer rows but never number more than bwd_bf16_max_groups
    w.part_db = static_cast<float *>(
        c.take(4 * nn * p->H * B * (size_t)tri::bwd_bf16_max_groups((int)p->N, p->H)));
  } else {
    w.part_db = w.ngroups > 1
                    ? static_cast<float *>(c.take(4 * nn * p->H * (size_t)w.ngroups))
                    : nullptr;
  }
  if (out) *out = w;
  return c.off;
}

// ------------------------------------------------------------ tensor maps --

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // The driver's encoder wants a current context on this host thread, which a
  // thread whose first CUDA work is a call into this library (a fresh thread,
  // or a worker whose allocations all came from a cache) may not have yet:
  // bind the runtime's primary context of the thread's current device.
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// A batch of pair tensors [batch][.., .., H, 32] bf16 seen through the frame;
// dimensions by increasing stride (c, h, the smaller of x/r, the larger, the
// problem), box = one 128 x 32 tile. The problem is a dimension of its own so
// that a tile reaching past N reads zeros, not the next problem.
bool encode_pair(CUtensorMap *m, const void *base, int64_t N, int64_t H, int64_t sR, int64_t sX,
                 bool x_inner, uint32_t box_rows = 128, int64_t batch = 1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[5] = {32, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)N, (cuuint64_t)batch};
  cuuint64_t strides[4] = {64, (cuuint64_t)((x_inner ? sX : sR) * 2),
                           (cuuint64_t)((x_inner ? sR : sX) * 2), (cuuint64_t)(N * N * H * 64)};
  cuuint32_t box[5] = {32, 1, x_inner ? box_rows : 1u, x_inner ? 1u : box_rows, 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Bias [H, N, N] bf16 in the variant frame (y fastest), box 64 keys x 128 queries.
bool encode_bias(CUtensorMap *m, const void *base, int64_t N, int64_t H, int64_t batch = 1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)N, (cuuint64_t)(H * batch)};
  cuuint64_t strides[2] = {(cuuint64_t)(N * 2), (cuuint64_t)(N * N * 2)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

tri_attn_status cuda_status(cudaError_t e);

// A dense stack [batch][rows][cols] (cols contiguous) as a 3-D tensor map with
// boxes of box_cols x box_rows and the 128-byte swizzle.
bool encode_stack(CUtensorMap *m, const void *base, bool f32, int64_t cols, int64_t rows,
                  int64_t batch, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int64_t es = f32 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)(cols * es), (cuuint64_t)(rows * cols * es)};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A GEMM operand whose product dimension has `mn` entries and whose summed
// dimension has `k`: K-major when stored [mn][k], MN-major when stored [k][mn].
bool encode_operand(CUtensorMap *m, const void *base, bool mn_major, int64_t mn, int64_t k,
                    int64_t batch) {
  return mn_major ? encode_stack(m, base, false, mn, k, batch, 64, 64)
                  : encode_stack(m, base, false, k, mn, batch, 64, 128);
}

// D = X Y^T per batch into one bf16 output [batch][M][Nn].
tri_attn_status gemm_bf16(const void *x, bool x_mn, const void *y, bool y_mn, void *out,
                          int64_t M, int64_t Nn, int64_t K, int64_t batch, int32_t *status,
                          cudaStream_t stream) {
  tri::GemmMaps ys;
  tri::GemmMaps xs;
  tri::GemmOuts outs;
  if (!encode_operand(&xs.map[0], x, x_mn, M, K, batch) ||
      !encode_operand(&ys.map[0], y, y_mn, Nn, K, batch) ||
      !encode_stack(&outs.map[0], out, false, Nn, M, batch, 64, 32))
    return TRI_ATTN_ERR_CUDA;
  tri::GemmArgs args{};
  args.M = (int)M;
  args.Nn = (int)Nn;
  args.K = (int)K;
  args.batch = (int)batch;
  args.nouts = 1;
  args.cols_per_out = (int)Nn;
  args.k_per_x = 1 << 30;           // one X tensor: every K slice comes from map 0
  args.col_bias = nullptr;
  args.status = status;
  return cuda_status(tri::launch_gemm_tc(x_mn, y_mn, false, xs, ys, outs, args, stream));
}

tri_attn_status check_mul(const tri_mul_problem *p) {
  if (!p) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->N < 0 || p->N > kMaxN || p->C < 1 || p->C > 65535) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->direction != TRI_MUL_OUTGOING && p->direction != TRI_MUL_INCOMING)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (p->N % 8 != 0) return TRI_ATTN_ERR_UNSUPPORTED;
  return TRI_ATTN_OK;
}

// One product D = X Y^T of the contraction (channel-major N x N per channel).
tri_attn_status mul_product(const tri_mul_problem *p, const void *x, bool x_mn, const void *y,
                            bool y_mn, void *out, int32_t *status, cudaStream_t stream) {
  return gemm_bf16(x, x_mn, y, y_mn, out, p->N, p->N, p->N, p->C, status, stream);
}

// The CUDA error behind the last TRI_ATTN_ERR_CUDA of this host thread.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

tri_attn_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return TRI_ATTN_OK;
  g_last_cuda_error = e;
  return TRI_ATTN_ERR_CUDA;
}

// Record the caller's timing event before (start) or after (stop) the main kernel.
// The residual tensor of the options (NULL when absent or past struct_size).
void *opt_residual(const tri_attn_launch_opts *opts) {
  if (!opts || opts->struct_size < offsetof(tri_attn_launch_opts, out_residual) + sizeof(void *))
    return nullptr;
  return opts->out_residual;
}

// Options are well formed: a known size, no flags beyond `allowed`, an aligned
// residual that only the bf16 path takes.
tri_attn_status check_opts(const tri_attn_problem *prob, const tri_attn_launch_opts *opts,
                           uint32_t allowed) {
  if (!opts) return TRI_ATTN_OK;
  if (opts->struct_size < TRI_ATTN_LAUNCH_OPTS_V1_SIZE || (opts->flags & ~allowed) != 0)
    return TRI_ATTN_ERR_INVALID_ARG;
  const void *res = opt_residual(opts);
  if (res && !aligned16(res)) return TRI_ATTN_ERR_INVALID_ARG;
  if (res && !tc_shape(prob)) return TRI_ATTN_ERR_UNSUPPORTED;
  return TRI_ATTN_OK;
}

cudaError_t mark(const tri_attn_launch_opts *opts, bool start, cudaStream_t stream) {
  if (!opts) return cudaSuccess;
  void *ev = start ? opts->main_start : opts->main_stop;
  if (!ev) return cudaSuccess;
  return cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev), stream);
}

#define TRI_CHECK_PTR(p)                                   \
  do {                                                     \
    if (!(p) || !aligned16(p)) return TRI_ATTN_ERR_INVALID_ARG; \
  } while (0)

}  // namespace

namespace {

// The CUDA-core kernels with the caller's tensors of type T.
template <typename T>
cudaError_t core_fwd(const Frame &f, const void *q, const void *k, const void *v,
                     const void *bias, const void *gate, void *out, float *lse,
                     cudaStream_t stream) {
  return tri::launch_f32_fwd<T>(f, static_cast<const T *>(q), static_cast<const T *>(k),
                                static_cast<const T *>(v), static_cast<const T *>(bias),
                                static_cast<const T *>(gate), static_cast<T *>(out), lse, stream);
}

template <typename T>
cudaError_t core_bwd(const Frame &f, const void *q, const void *k, const void *v,
                     const void *bias, const void *gate, const void *out, const float *lse,
                     const void *dout, void *dq, void *dk, void *dv, void *dbias, void *dgate,
                     const tri::F32BwdScratch &s, cudaStream_t stream) {
  return tri::launch_f32_bwd<T>(f, static_cast<const T *>(q), static_cast<const T *>(k),
                                static_cast<const T *>(v), static_cast<const T *>(bias),
                                static_cast<const T *>(gate), static_cast<const T *>(out), lse,
                                static_cast<const T *>(dout), static_cast<T *>(dq),
                                static_cast<T *>(dk), static_cast<T *>(dv),
                                static_cast<T *>(dbias), static_cast<T *>(dgate), s, stream);
}

}  // namespace

extern "C" {

int tri_attn_version(void) { return (1 << 16) | 0; }

const char *tri_attn_last_cuda_error(void) {
  return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

const char *tri_attn_status_string(tri_attn_status s) {
  switch (s) {
    case TRI_ATTN_OK: return "ok";
    case TRI_ATTN_ERR_INVALID_ARG: return "invalid argument";
    case TRI_ATTN_ERR_UNSUPPORTED: return "unsupported problem";
    case TRI_ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case TRI_ATTN_ERR_CUDA: return "CUDA call failed";
    case TRI_ATTN_ERR_TIMEOUT: return "device wait timed out";
    case TRI_ATTN_ERR_BOUNDS: return "device index check failed";
  }
  return "unknown status";
}

tri_attn_status tri_attn_fwd_workspace_size(const tri_attn_problem *prob, size_t *bytes) {
  tri_attn_status st = check_problem(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!bytes) return TRI_ATTN_ERR_INVALID_ARG;
  *bytes = carve_fwd(prob, nullptr, true, nullptr);
  return TRI_ATTN_OK;
}

tri_attn_status tri_attn_bwd_workspace_size(const tri_attn_problem *prob, size_t *bytes) {
  tri_attn_status st = check_problem(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!bytes) return TRI_ATTN_ERR_INVALID_ARG;
  // large enough for either backward path (TRI_ATTN_OPT_ONCHIP_SUMS or not)
  *bytes = std::max(carve_bwd(prob, nullptr, true, false, nullptr),
                    carve_bwd(prob, nullptr, true, true, nullptr));
  return TRI_ATTN_OK;
}

namespace {

// Forward over the attention rows [row0, row0 + row_count) (validated by the caller).
tri_attn_status fwd_impl(const tri_attn_problem *prob, const void *q, const void *k,
                         const void *v, const void *bias, const void *gate, const uint8_t *mask,
                         void *out, float *lse, void *workspace, size_t workspace_bytes,
                         tri_attn_stream_t stream_, const tri_attn_launch_opts *opts,
                         int64_t row0, int64_t row_count) {
  tri_attn_status st = check_problem(prob);
  if (st != TRI_ATTN_OK) return st;
  st = check_opts(prob, opts, TRI_ATTN_OPT_EXP2_SPLIT);
  if (st != TRI_ATTN_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return TRI_ATTN_ERR_WORKSPACE;
  const bool per_row = mask && prob->mask_row_stride == prob->N;
  FwdWs w;
  if (workspace_bytes < carve_fwd(prob, workspace, per_row, &w)) return TRI_ATTN_ERR_WORKSPACE;
  if (prob->N == 0) return TRI_ATTN_OK;
  TRI_CHECK_PTR(q); TRI_CHECK_PTR(k); TRI_CHECK_PTR(v); TRI_CHECK_PTR(bias);
  TRI_CHECK_PTR(gate); TRI_CHECK_PTR(out); TRI_CHECK_PTR(lse);
  Frame f = make_frame(prob, mask, w.status);
  const bool whole = row_count < 0;                  // every row of every problem
  if (whole) row_count = f.row_end;
  f.row0 = (int)row0;
  f.row_end = (int)(row0 + row_count);
  if (row_count == 0) return TRI_ATTN_OK;

  if (!tc_shape(prob)) {
    // CUDA-core kernels (fp32, or bf16 storage with fp32 arithmetic), one
    // problem of the batch after another
    if (!whole) return TRI_ATTN_ERR_UNSUPPORTED;
    cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(int32_t), stream);
    if (e == cudaSuccess) e = mark(opts, true, stream);
    const ProblemStrides ps = problem_strides(prob, mask != nullptr);
    for (int64_t b = 0; e == cudaSuccess && b < batch_of(prob); ++b) {
      Frame fb = make_frame(prob, mask ? mask + b * ps.mask : nullptr, w.status);
      fb.B = 1;
      fb.row_end = f.N;
      e = prob->dtype == TRI_ATTN_F32
              ? core_fwd<float>(fb, at(q, b * ps.pair), at(k, b * ps.pair), at(v, b * ps.pair),
                                at(bias, b * ps.bias), at(gate, b * ps.pair), at(out, b * ps.pair),
                                lse + b * ps.lse, stream)
              : core_fwd<__nv_bfloat16>(fb, at(q, b * ps.pair), at(k, b * ps.pair),
                                        at(v, b * ps.pair), at(bias, b * ps.bias),
                                        at(gate, b * ps.pair), at(out, b * ps.pair),
                                        lse + b * ps.lse, stream);
    }
    if (e == cudaSuccess) e = mark(opts, false, stream);
    return cuda_status(e);
  }

  const int64_t words = mask_words_per_row(prob);
  const int64_t rows = mask_rows(prob, mask != nullptr);
  const bool x_inner = prob->variant == TRI_ATTN_STARTING;
  tri::FwdMaps maps;
  const void *bias_frame = prob->variant == TRI_ATTN_ENDING ? w.biasT : bias;
  const uint32_t kv_rows = (uint32_t)tri::fwd_bf16_key_tile();
  const int64_t B = f.B;
  if (!encode_pair(&maps.q, q, prob->N, prob->H, f.sR, f.sX, x_inner, 128, B) ||
      !encode_pair(&maps.k, k, prob->N, prob->H, f.sR, f.sX, x_inner, kv_rows, B) ||
      !encode_pair(&maps.v, v, prob->N, prob->H, f.sR, f.sX, x_inner, kv_rows, B) ||
      !encode_bias(&maps.bias, bias_frame, prob->N, prob->H, B))
    return TRI_ATTN_ERR_CUDA;
  tri::FwdArgs a;
  a.N = f.N;
  a.H = f.H;
  a.row0 = f.row0;
  a.row_end = f.row_end;
  a.exp2_split = (opts && (opts->flags & TRI_ATTN_OPT_EXP2_SPLIT)) ? 1 : 0;
  a.x_inner = x_inner ? 1 : 0;
  a.scale = 1.0f / sqrtf((float)prob->c);
  a.sR = f.sR;
  a.sX = f.sX;
  a.gate = static_cast<const __nv_bfloat16 *>(gate);
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.out_res = static_cast<__nv_bfloat16 *>(opt_residual(opts));
  a.lse = lse;
  a.mask_bits = w.mask_bits;
  a.mask_bits_stride = words;
  a.mask_per_row = per_row ? 1 : 0;
  a.status = w.status;
  cudaError_t e =
      tri::launch_mask_bits(f, w.mask_bits, rows, words, w.status, nullptr, 0, stream);
  if (e == cudaSuccess && prob->variant == TRI_ATTN_ENDING)
    e = tri::launch_bias_transpose(static_cast<const __nv_bfloat16 *>(bias), w.biasT, f.N,
                                   f.H * f.B, stream);
  if (e == cudaSuccess) e = mark(opts, true, stream);
  if (e == cudaSuccess) e = tri::launch_fwd_bf16(maps, a, stream);
  if (e == cudaSuccess) e = mark(opts, false, stream);
  return cuda_status(e);
}

}  // namespace

tri_attn_status tri_attn_fwd_ex(const tri_attn_problem *prob, const void *q, const void *k,
                                const void *v, const void *bias, const void *gate,
                                const uint8_t *mask, void *out, float *lse, void *workspace,
                                size_t workspace_bytes, tri_attn_stream_t stream,
                                const tri_attn_launch_opts *opts) {
  return fwd_impl(prob, q, k, v, bias, gate, mask, out, lse, workspace, workspace_bytes, stream,
                  opts, 0, -1);
}

tri_attn_status tri_attn_fwd(const tri_attn_problem *prob, const void *q, const void *k,
                             const void *v, const void *bias, const void *gate,
                             const uint8_t *mask, void *out, float *lse, void *workspace,
                             size_t workspace_bytes, tri_attn_stream_t stream) {
  return tri_attn_fwd_ex(prob, q, k, v, bias, gate, mask, out, lse, workspace, workspace_bytes,
                         stream, nullptr);
}

namespace {

// Backward over the attention rows [row0, row0 + row_count) (validated by the
// caller). dbias_partial != NULL: the fp32 sum of dbias over these rows goes
// there instead of the bf16 dbias.
tri_attn_status bwd_impl(const tri_attn_problem *prob, const void *q, const void *k,
                         const void *v, const void *bias, const void *gate, const uint8_t *mask,
                         const void *out, const float *lse, const void *dout, void *dq, void *dk,
                         void *dv, void *dbias, float *dbias_partial, void *dgate,
                         void *workspace, size_t workspace_bytes, tri_attn_stream_t stream_,
                         const tri_attn_launch_opts *opts, int64_t row0, int64_t row_count) {
  tri_attn_status st = check_problem(prob);
  if (st != TRI_ATTN_OK) return st;
  st = check_opts(prob, opts, TRI_ATTN_OPT_ONCHIP_SUMS);
  if (st != TRI_ATTN_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return TRI_ATTN_ERR_WORKSPACE;
  const bool per_row = mask && prob->mask_row_stride == prob->N;
  const bool onchip = opts && (opts->flags & TRI_ATTN_OPT_ONCHIP_SUMS) != 0;
  if (onchip && prob->dtype != TRI_ATTN_BF16) return TRI_ATTN_ERR_INVALID_ARG;
  // (bf16 shapes of the CUDA-core kernels take the default path)
  BwdWs w;
  if (workspace_bytes < carve_bwd(prob, workspace, per_row, onchip, &w))
    return TRI_ATTN_ERR_WORKSPACE;
  if (prob->N == 0) return TRI_ATTN_OK;
  TRI_CHECK_PTR(q); TRI_CHECK_PTR(k); TRI_CHECK_PTR(v); TRI_CHECK_PTR(bias);
  TRI_CHECK_PTR(gate); TRI_CHECK_PTR(out); TRI_CHECK_PTR(lse); TRI_CHECK_PTR(dout);
  TRI_CHECK_PTR(dq); TRI_CHECK_PTR(dk); TRI_CHECK_PTR(dv); TRI_CHECK_PTR(dgate);
  if (dbias_partial) {
    TRI_CHECK_PTR(dbias_partial);
  } else {
    TRI_CHECK_PTR(dbias);
  }
  Frame f = make_frame(prob, mask, w.fw.status);
  const bool whole = row_count < 0;                  // every row of every problem
  if (whole) row_count = f.row_end;
  f.row0 = (int)row0;
  f.row_end = (int)(row0 + row_count);
  const bool shard = dbias_partial != nullptr || !whole;
  if (row_count == 0) return TRI_ATTN_OK;

  if (!tc_shape(prob)) {
    // CUDA-core kernels (fp32, or bf16 storage with fp32 arithmetic), one
    // problem of the batch after another on the same scratch
    if (shard) return TRI_ATTN_ERR_UNSUPPORTED;
    tri::F32BwdScratch s;
    s.du = static_cast<float *>(w.du);
    s.D = w.D;
    s.part_dq = w.part_dq;
    s.part_dk = w.part_dk;
    s.part_dv = w.part_dv;
    s.part_db = w.part_db;
    s.ntile = w.ntile;
    s.ngroups = w.ngroups;
    cudaError_t e = cudaMemsetAsync(w.fw.status, 0, sizeof(int32_t), stream);
    if (e == cudaSuccess) e = mark(opts, true, stream);
    const ProblemStrides ps = problem_strides(prob, mask != nullptr);
    for (int64_t b = 0; e == cudaSuccess && b < batch_of(prob); ++b) {
      Frame fb = make_frame(prob, mask ? mask + b * ps.mask : nullptr, w.fw.status);
      fb.B = 1;
      fb.row_end = f.N;
      const int64_t o = b * ps.pair;
      e = prob->dtype == TRI_ATTN_F32
              ? core_bwd<float>(fb, at(q, o), at(k, o), at(v, o), at(bias, b * ps.bias),
                                at(gate, o), at(out, o), lse + b * ps.lse, at(dout, o), at(dq, o),
                                at(dk, o), at(dv, o), at(dbias, b * ps.bias), at(dgate, o), s,
                                stream)
              : core_bwd<__nv_bfloat16>(fb, at(q, o), at(k, o), at(v, o), at(bias, b * ps.bias),
                                        at(gate, o), at(out, o), lse + b * ps.lse, at(dout, o),
                                        at(dq, o), at(dk, o), at(dv, o), at(dbias, b * ps.bias),
                                        at(dgate, o), s, stream);
    }
    if (e == cudaSuccess) e = mark(opts, false, stream);
    return cuda_status(e);
  }

  const int64_t words = mask_words_per_row(prob);
  const int64_t rows = mask_rows(prob, mask != nullptr);
  const bool x_inner = prob->variant == TRI_ATTN_STARTING;
  const int64_t N = prob->N, H = prob->H;
  const float scale = 1.0f / sqrtf((float)prob->c);

  if (w.tc && !shard) {
    tri::BwdMaps maps;
    if (!encode_pair(&maps.q, q, N, H, f.sR, f.sX, x_inner) ||
        !encode_pair(&maps.k, k, N, H, f.sR, f.sX, x_inner) ||
        !encode_pair(&maps.v, v, N, H, f.sR, f.sX, x_inner) ||
        !encode_pair(&maps.du, w.du, N, H, N * H * 32, H * 32, true))
      return TRI_ATTN_ERR_CUDA;
    tri::BwdTcArgs a{};
    a.N = f.N;
    a.H = f.H;
    a.x_inner = x_inner ? 1 : 0;
    a.nb = w.ntile;
    a.ngroups = w.ngroups;
    a.rows_per_group = (f.N + w.ngroups - 1) / w.ngroups;
    a.scale = scale;
    a.sR = f.sR;
    a.sX = f.sX;
    a.bX = f.bX;
    a.bY = f.bY;
    a.bias = static_cast<const __nv_bfloat16 *>(bias);
    a.LD = reinterpret_cast<const float4 *>(w.LD);
    a.mask_bits = w.fw.mask_bits;
    a.mask_bits_stride = rows > 1 ? words : 0;
    a.dq = static_cast<__nv_bfloat16 *>(dq);
    a.dk = static_cast<__nv_bfloat16 *>(dk);
    a.dv = static_cast<__nv_bfloat16 *>(dv);
    a.dbias = static_cast<__nv_bfloat16 *>(dbias);
    a.part_db = w.part_db;
    a.ring = w.ring;
    const int64_t gh_total = (int64_t)w.ngroups * H, nb = w.ntile;
    a.exported = w.flags;
    a.consumed_q = w.flags + gh_total * nb * nb;
    a.consumed_kv = a.consumed_q + gh_total * nb * tri::bwd_tc_consumed_flags_per_tile();
    a.status = w.fw.status;
    // mask bits, status reset and the exchange flags zeroed in one launch
    cudaError_t e = tri::launch_mask_bits(f, w.fw.mask_bits, rows, words, w.fw.status, w.flags,
                                          w.nflags, stream);
    if (e == cudaSuccess)
      e = tri::launch_bwd_pre_bf16(f, static_cast<const __nv_bfloat16 *>(gate),
                                   static_cast<const __nv_bfloat16 *>(out),
                                   static_cast<const __nv_bfloat16 *>(opt_residual(opts)),
                                   static_cast<const __nv_bfloat16 *>(dout),
                                   static_cast<__nv_bfloat16 *>(w.du), nullptr,
                                   static_cast<__nv_bfloat16 *>(dgate), lse, w.LD, stream);
    if (e == cudaSuccess) e = mark(opts, true, stream);
    for (int64_t gh0 = 0; e == cudaSuccess && gh0 < gh_total; gh0 += w.ghl) {
      a.gh0 = (int)gh0;
      a.ghl = (int)std::min<int64_t>(w.ghl, gh_total - gh0);
      e = tri::launch_bwd_tc(maps, a, stream);
    }
    if (e == cudaSuccess) e = mark(opts, false, stream);
    if (e == cudaSuccess && w.ngroups > 1)
      e = tri::launch_bias_reduce<__nv_bfloat16>(f, w.part_db, w.ngroups,
                                                 static_cast<__nv_bfloat16 *>(dbias), stream);
    return cuda_status(e);
  }

  const void *bias_frame = prob->variant == TRI_ATTN_ENDING ? w.fw.biasT : bias;
  tri::BwdMaps maps;
  const int64_t B = f.B;
  if (!encode_pair(&maps.q, q, N, H, f.sR, f.sX, x_inner, 128, B) ||
      !encode_pair(&maps.k, k, N, H, f.sR, f.sX, x_inner, 128, B) ||
      !encode_pair(&maps.v, v, N, H, f.sR, f.sX, x_inner, 128, B) ||
      !encode_pair(&maps.du, w.du, N, H, N * H * 32, H * 32, true, 128, B) ||
      !encode_bias(&maps.bias, bias_frame, N, H, B))
    return TRI_ATTN_ERR_CUDA;
  // row groups of each problem's rows (a row shard's rows when B = 1), planned
  // as for the problem alone: each problem of a batch gets the results, bit for
  // bit, that a call on it alone gives
  const int64_t rows_per_problem = whole ? N : row_count;
  int ntile = w.ntile, ngroups = w.ngroups;
  tri::bwd_bf16_plan(f.N, f.H, (int)rows_per_problem, &ntile, &ngroups);
  tri::BwdArgs a;
  a.N = f.N;
  a.H = f.H;
  a.B = f.B;
  a.row0 = f.row0;
  a.row_end = f.row_end;
  a.x_inner = x_inner ? 1 : 0;
  a.nb = ntile;
  a.scale = scale;
  a.sR = f.sR;
  a.sX = f.sX;
  a.lse = lse;
  a.D = w.D;
  a.mask_bits = w.fw.mask_bits;
  a.mask_bits_stride = words;
  a.mask_per_row = per_row ? 1 : 0;
  a.part_q = w.bpart_q;
  a.part_k = w.bpart_k;
  a.part_v = w.bpart_v;
  a.part_db = w.part_db;
  // one row group over every row writes dbias itself; otherwise per-group fp32 sums
  a.dbias = (!dbias_partial && ngroups == 1) ? static_cast<__nv_bfloat16 *>(dbias) : nullptr;
  a.bX = f.bX;
  a.bY = f.bY;
  a.ngroups = ngroups;
  a.rows_per_group = (int)((rows_per_problem + ngroups - 1) / ngroups);
  a.status = w.fw.status;

  cudaError_t e = tri::launch_mask_bits(f, w.fw.mask_bits, rows, words, w.fw.status, nullptr,
                                        0, stream);
  if (e == cudaSuccess && prob->variant == TRI_ATTN_ENDING)
    e = tri::launch_bias_transpose(static_cast<const __nv_bfloat16 *>(bias), w.fw.biasT, f.N,
                                   f.H * f.B, stream);
  if (e == cudaSuccess)
    e = tri::launch_bwd_pre_bf16(f, static_cast<const __nv_bfloat16 *>(gate),
                                 static_cast<const __nv_bfloat16 *>(out),
                                 static_cast<const __nv_bfloat16 *>(opt_residual(opts)),
                                 static_cast<const __nv_bfloat16 *>(dout),
                                 static_cast<__nv_bfloat16 *>(w.du), w.D,
                                 static_cast<__nv_bfloat16 *>(dgate), nullptr, nullptr, stream);
  if (e == cudaSuccess) e = mark(opts, true, stream);
  if (e == cudaSuccess) e = tri::launch_bwd_bf16(maps, a, stream);
  if (e == cudaSuccess) e = mark(opts, false, stream);
  if (e == cudaSuccess)
    e = tri::launch_partial_reduce_bf16(f, w.bpart_q, w.bpart_k, w.bpart_v, w.ntile, a.scale,
                                        static_cast<__nv_bfloat16 *>(dq),
                                        static_cast<__nv_bfloat16 *>(dk),
                                        static_cast<__nv_bfloat16 *>(dv), stream);
  // the per-group sums are [group][B*H][N][N]: the reduction sees B*H heads
  Frame fh = f;
  fh.H = f.H * f.B;
  if (e == cudaSuccess && dbias_partial)
    e = tri::launch_bias_reduce<float>(fh, w.part_db, ngroups, dbias_partial, stream);
  else if (e == cudaSuccess && ngroups > 1)
    e = tri::launch_bias_reduce<__nv_bfloat16>(fh, w.part_db, ngroups,
                                               static_cast<__nv_bfloat16 *>(dbias), stream);
  return cuda_status(e);
}

}  // namespace

tri_attn_status tri_attn_bwd_ex(const tri_attn_problem *prob, const void *q, const void *k,
                                const void *v, const void *bias, const void *gate,
                                const uint8_t *mask, const void *out, const float *lse,
                                const void *dout, void *dq, void *dk, void *dv, void *dbias,
                                void *dgate, void *workspace, size_t workspace_bytes,
                                tri_attn_stream_t stream, const tri_attn_launch_opts *opts) {
  return bwd_impl(prob, q, k, v, bias, gate, mask, out, lse, dout, dq, dk, dv, dbias, nullptr,
                  dgate, workspace, workspace_bytes, stream, opts, 0, -1);
}

namespace {
// A row shard is a whole number of 8-row groups inside [0, N).
tri_attn_status check_rows(const tri_attn_problem *prob, int64_t row_begin, int64_t row_count) {
  if (!prob || row_begin < 0 || row_count < 0 || row_begin + row_count > prob->N)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (row_begin % 8 != 0 || row_count % 8 != 0) return TRI_ATTN_ERR_INVALID_ARG;
  return TRI_ATTN_OK;
}
}  // namespace

tri_attn_status tri_attn_fwd_rows(const tri_attn_problem *prob, int64_t row_begin,
                                  int64_t row_count, const void *q, const void *k, const void *v,
                                  const void *bias, const void *gate, const uint8_t *mask,
                                  void *out, float *lse, void *workspace, size_t workspace_bytes,
                                  tri_attn_stream_t stream) {
  tri_attn_status st = check_problem(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!tc_shape(prob) || batch_of(prob) != 1) return TRI_ATTN_ERR_UNSUPPORTED;
  st = check_rows(prob, row_begin, row_count);
  if (st != TRI_ATTN_OK) return st;
  return fwd_impl(prob, q, k, v, bias, gate, mask, out, lse, workspace, workspace_bytes, stream,
                  nullptr, row_begin, row_count);
}

tri_attn_status tri_attn_bwd_rows(const tri_attn_problem *prob, int64_t row_begin,
                                  int64_t row_count, const void *q, const void *k, const void *v,
                                  const void *bias, const void *gate, const uint8_t *mask,
                                  const void *out, const float *lse, const void *dout, void *dq,
                                  void *dk, void *dv, float *dbias_partial, void *dgate,
                                  void *workspace, size_t workspace_bytes,
                                  tri_attn_stream_t stream) {
  tri_attn_status st = check_problem(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!tc_shape(prob) || batch_of(prob) != 1) return TRI_ATTN_ERR_UNSUPPORTED;
  st = check_rows(prob, row_begin, row_count);
  if (st != TRI_ATTN_OK) return st;
  if (!dbias_partial && prob->N > 0) return TRI_ATTN_ERR_INVALID_ARG;
  return bwd_impl(prob, q, k, v, bias, gate, mask, out, lse, dout, dq, dk, dv, nullptr,
                  dbias_partial, dgate, workspace, workspace_bytes, stream, nullptr, row_begin,
                  row_count);
}

tri_attn_status tri_attn_dbias_reduce(const float *partials, int32_t count, int64_t N, int32_t H,
                                      void *dbias, tri_attn_stream_t stream) {
  if (count < 1 || N < 0 || N > kMaxN || H < 1 || (N > 0 && (!partials || !dbias)))
    return TRI_ATTN_ERR_INVALID_ARG;
  if (!aligned16(partials) || !aligned16(dbias)) return TRI_ATTN_ERR_INVALID_ARG;
  if (N == 0) return TRI_ATTN_OK;
  // the partials and dbias share one [H][N][N] layout: an identity frame
  Frame f{};
  f.N = (int)N;
  f.H = H;
  f.B = 1;
  f.bX = N;
  f.bY = 1;
  return cuda_status(tri::launch_bias_reduce<__nv_bfloat16>(
      f, partials, count, static_cast<__nv_bfloat16 *>(dbias),
      reinterpret_cast<cudaStream_t>(stream)));
}

tri_attn_status tri_attn_bwd(const tri_attn_problem *prob, const void *q, const void *k,
                             const void *v, const void *bias, const void *gate,
                             const uint8_t *mask, const void *out, const float *lse,
                             const void *dout, void *dq, void *dk, void *dv, void *dbias,
                             void *dgate, void *workspace, size_t workspace_bytes,
                             tri_attn_stream_t stream) {
  return tri_attn_bwd_ex(prob, q, k, v, bias, gate, mask, out, lse, dout, dq, dk, dv, dbias,
                         dgate, workspace, workspace_bytes, stream, nullptr);
}

tri_attn_status tri_attn_kernel_launches(const tri_attn_problem *prob, int backward,
                                         int has_mask, int32_t *launches) {
  tri_attn_status st = check_problem(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!launches || backward < 0 || backward > 2) return TRI_ATTN_ERR_INVALID_ARG;
  (void)has_mask;
  const bool onchip = backward == 2;
  int32_t n = 0;
  if (prob->N > 0) {
    if (!tc_shape(prob)) {
      // one problem of the batch after another
      const int32_t B = (int32_t)batch_of(prob);
      if (!backward) {
        n = B;
      } else {
        BwdWs w;
        carve_bwd(prob, nullptr, false, false, &w);
        n = B * (5 + (w.ngroups > 1 ? 1 : 0));  // pre, main, three reductions, dbias reduction
      }
    } else {
      const int ending = prob->variant == TRI_ATTN_ENDING ? 1 : 0;
      if (!backward) {
        n = 2 + ending;  // mask bits, [bias transpose], main
      } else {
        BwdWs w;
        carve_bwd(prob, nullptr, false, onchip, &w);
        if (w.tc) {
          // mask bits, pre, one main launch per group of (group, head) pairs,
          // [dbias reduction]
          const int64_t gh = (int64_t)w.ngroups * prob->H;
          n = 2 + (int32_t)((gh + w.ghl - 1) / w.ghl) + (w.ngroups > 1 ? 1 : 0);
        } else {
          // mask bits, [transpose], pre, main, partial reduction, [dbias reduction]
          n = 4 + ending + (w.ngroups > 1 ? 1 : 0);
        }
      }
    }
  }
  *launches = n;
  return TRI_ATTN_OK;
}

tri_attn_status tri_attn_read_status(const void *workspace, int32_t *device_status,
                                     tri_attn_stream_t stream_) {
  if (!workspace || !device_status) return TRI_ATTN_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int32_t v = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return TRI_ATTN_ERR_CUDA;
  *device_status = v;
  return TRI_ATTN_OK;
}

tri_attn_status tri_attn_get_status(const void *workspace, tri_attn_stream_t stream) {
  int32_t v = 0;
  const tri_attn_status st = tri_attn_read_status(workspace, &v, stream);
  return st != TRI_ATTN_OK ? st : static_cast<tri_attn_status>(v);
}

tri_attn_status tri_attn_check_exp2(const float *x, float *y_fma, float *y_mufu, int64_t n,
                                    tri_attn_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y_fma || !y_mufu))) return TRI_ATTN_ERR_INVALID_ARG;
  return cuda_status(
      tri::launch_exp2_eval(x, y_fma, y_mufu, n, reinterpret_cast<cudaStream_t>(stream)));
}

tri_attn_status tri_attn_probe_mma(int32_t n, int32_t layout, int32_t ctas, int32_t instructions,
                                   unsigned long long *cycles, int32_t *status,
                                   tri_attn_stream_t stream) {
  const bool n_ok = n == 32 || n == 64 || n == 128 || n == 256;
  if (!n_ok || layout < 0 || layout > 2 || (layout != 0 && n != 32) || ctas < 1 ||
      ctas > 1024 || instructions < 1 || instructions > (1 << 24) || !cycles || !status)
    return TRI_ATTN_ERR_INVALID_ARG;
  return cuda_status(tri::launch_mma_probe(n, layout, ctas, instructions, cycles, status,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

tri_attn_status tri_attn_check_wait_timeout(void *workspace, size_t workspace_bytes,
                                            tri_attn_stream_t stream) {
  if (!workspace || !aligned16(workspace) || workspace_bytes < 256)
    return TRI_ATTN_ERR_WORKSPACE;
  return cuda_status(tri::launch_unsatisfied_wait(static_cast<int32_t *>(workspace),
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

tri_attn_status tri_mul_workspace_size(const tri_mul_problem *prob, size_t *bytes) {
  tri_attn_status st = check_mul(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!bytes) return TRI_ATTN_ERR_INVALID_ARG;
  *bytes = 256;
  return TRI_ATTN_OK;
}

tri_attn_status tri_mul_fwd(const tri_mul_problem *prob, const void *a, const void *b, void *t,
                            void *workspace, size_t workspace_bytes, tri_attn_stream_t stream_) {
  tri_attn_status st = check_mul(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!workspace || !aligned16(workspace) || workspace_bytes < 256) return TRI_ATTN_ERR_WORKSPACE;
  TRI_CHECK_PTR(a);
  TRI_CHECK_PTR(b);
  TRI_CHECK_PTR(t);
  if (prob->N == 0) return TRI_ATTN_OK;      // nothing to do, nothing enqueued
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int32_t *status = static_cast<int32_t *>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), stream) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  // outgoing: t = A B^T (both K-major); incoming: t = A^T B (both MN-major)
  const bool mn = prob->direction == TRI_MUL_INCOMING;
  return mul_product(prob, a, mn, b, mn, t, status, stream);
}

tri_attn_status tri_mul_bwd(const tri_mul_problem *prob, const void *a, const void *b,
                            const void *dt, void *da, void *db, void *workspace,
                            size_t workspace_bytes, tri_attn_stream_t stream_) {
  tri_attn_status st = check_mul(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!workspace || !aligned16(workspace) || workspace_bytes < 256) return TRI_ATTN_ERR_WORKSPACE;
  TRI_CHECK_PTR(a);
  TRI_CHECK_PTR(b);
  TRI_CHECK_PTR(dt);
  TRI_CHECK_PTR(da);
  TRI_CHECK_PTR(db);
  if (prob->N == 0) return TRI_ATTN_OK;      // nothing to do, nothing enqueued
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int32_t *status = static_cast<int32_t *>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), stream) != cudaSuccess) return TRI_ATTN_ERR_CUDA;
  if (prob->direction == TRI_MUL_OUTGOING) {
    // da[i][k] = sum_j dt[i][j] b[j][k];  db[j][k] = sum_i dt[i][j] a[i][k]
    st = mul_product(prob, dt, false, b, true, da, status, stream);
    if (st == TRI_ATTN_OK) st = mul_product(prob, dt, true, a, true, db, status, stream);
  } else {
    // da[k][i] = sum_j b[k][j] dt[i][j];  db[k][j] = sum_i a[k][i] dt[i][j]
    st = mul_product(prob, b, false, dt, false, da, status, stream);
    if (st == TRI_ATTN_OK) st = mul_product(prob, a, false, dt, true, db, status, stream);
  }
  return st;
}

}  // extern "C"

// ------------------------------------------------ LayerNorm and projections --

namespace {

constexpr int kGemmTileM = 128, kGemmTileN = 256, kGemmTileK = 64;
constexpr int kSplitTargetCtas = 2 * 148;      // two CTAs per SM

int64_t proj_total_rows(const tri_proj_problem *p) { return p->rows * (int64_t)p->batch; }

tri_attn_status check_proj(const tri_proj_problem *p) {
  if (!p) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->rows < 0 || p->batch < 0 || p->cz < 1 || p->H < 1 || p->c < 1 || !(p->eps > 0.0f) ||
      !std::isfinite(p->eps) || p->reserved != 0)
    return TRI_ATTN_ERR_INVALID_ARG;
  if (p->cz % 64 || p->cz > 256 || p->H > 8 || p->c > 256 || (p->H * p->c) % 64 ||
      p->H * p->c > 256)
    return TRI_ATTN_ERR_UNSUPPORTED;
  if (p->rows > 0 && p->batch > 0 && proj_total_rows(p) >= (int64_t(1) << 31))
    return TRI_ATTN_ERR_UNSUPPORTED;
  return TRI_ATTN_OK;
}

// Split of a weight-gradient product (M x Nn, summed over K rows) into batches
// of k_split rows (a multiple of the 64-row K step) so that the grid fills two
// CTAs per SM; every batch gets at least one row.
struct KSplit {
  int k_split, n;
};
KSplit split_k(int64_t M, int64_t Nn, int64_t K) {
  const int64_t tiles = ((M + kGemmTileM - 1) / kGemmTileM) * ((Nn + kGemmTileN - 1) / kGemmTileN);
  int64_t s = kSplitTargetCtas / tiles;
  if (s < 1) s = 1;
  int64_t ks = (K + s - 1) / s;
  ks = (ks + kGemmTileK - 1) / kGemmTileK * kGemmTileK;
  if (ks < kGemmTileK) ks = kGemmTileK;
  return {(int)ks, (int)((K + ks - 1) / ks)};
}

struct ProjWs {
  int32_t *status;
  float *dx;      // [R][cz] fp32
  float *part;    // partial sums
};

// Workspace: the status word, dx, and the largest set of partial sums.
size_t carve_proj(const tri_proj_problem *p, void *base, ProjWs *ws) {
  const int64_t R = proj_total_rows(p), cz = p->cz, hc = (int64_t)p->H * p->c;
  const int64_t warps = tri::proj_partials();
  // input backward: LayerNorm partials then the db_g column-sum partials, or the
  // dW_qkvg split-K partials; output backward: the dW_o split-K partials then the
  // db_o column-sum partials
  int64_t part = warps * (cz * (2 + p->H) + hc);
  if (R > 0) {
    const KSplit si = split_k(cz, 4 * hc, R), so = split_k(hc, cz, R);
    part = std::max(part, (int64_t)si.n * cz * 4 * hc);
    part = std::max(part, (int64_t)so.n * hc * cz + warps * cz);
  }
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + kAlign - 1) / kAlign * kAlign;
    return o;
  };
  const size_t o_status = take(sizeof(int32_t));
  const size_t o_dx = take((size_t)R * cz * sizeof(float));
  const size_t o_part = take((size_t)part * sizeof(float));
  if (ws && base) {
    char *b = static_cast<char *>(base);
    ws->status = reinterpret_cast<int32_t *>(b + o_status);
    ws->dx = reinterpret_cast<float *>(b + o_dx);
    ws->part = reinterpret_cast<float *>(b + o_part);
  }
  return off;
}

tri_attn_status proj_begin(const tri_proj_problem *p, void *workspace, size_t workspace_bytes,
                           ProjWs *ws) {
  tri_attn_status st = check_proj(p);
  if (st != TRI_ATTN_OK) return st;
  if (!workspace || !aligned16(workspace) || workspace_bytes < carve_proj(p, nullptr, nullptr))
    return TRI_ATTN_ERR_WORKSPACE;
  carve_proj(p, workspace, ws);
  return TRI_ATTN_OK;
}

tri_attn_status zero_f32(float *p, size_t n, cudaStream_t s) {
  return cuda_status(cudaMemsetAsync(p, 0, n * sizeof(float), s));
}

// fp32 weight gradient D[M][Nn] = sum over the K rows of X[k][m] Y[k][n], X
// stored [K][M], Y as ny tensors [K][Nn / ny] side by side along n: split-K
// partials into ws->part, then one ordered sum into out [M][Nn].
tri_attn_status weight_grad(const void *x, const void *const *y, int ny, int64_t M, int64_t Nn,
                            int64_t K, float *out, const ProjWs &ws, cudaStream_t stream,
                            tri::SumSeg *defer = nullptr) {
  const KSplit sp = split_k(M, Nn, K);
  const int64_t per_y = Nn / ny;
  tri::GemmMaps xs, ys;
  tri::GemmOuts outs;
  if (!encode_operand(&xs.map[0], x, true, M, K, 1) ||
      !encode_stack(&outs.map[0], ws.part, true, Nn, M, sp.n, 32, 32))
    return TRI_ATTN_ERR_CUDA;
  for (int i = 0; i < ny; ++i)
    if (!encode_operand(&ys.map[i], y[i], true, per_y, K, 1)) return TRI_ATTN_ERR_CUDA;
  tri::GemmArgs args{};
  args.M = (int)M;
  args.Nn = (int)Nn;
  args.K = (int)K;
  args.batch = sp.n;
  args.nouts = 1;
  args.cols_per_out = (int)Nn;
  args.k_per_x = 1 << 30;
  args.n_per_y = ny > 1 ? (int)per_y : 0;
  args.ny = ny;
  args.k_split = sp.k_split;
  args.status = ws.status;
  tri_attn_status st = cuda_status(tri::launch_gemm_tc(true, true, true, xs, ys, outs, args, stream));
  if (st != TRI_ATTN_OK) return st;
  const tri::SumSeg seg{ws.part, sp.n, M * Nn, M * Nn, out, M * Nn, M * Nn};
  if (defer) {                 // the caller sums it together with other partials
    *defer = seg;
    return TRI_ATTN_OK;
  }
  return cuda_status(tri::launch_ordered_sums(&seg, 1, stream));
}

// Elements of the split-K partials of a weight gradient (where other partials
// may follow in the workspace).
int64_t weight_grad_partials(int64_t M, int64_t Nn, int64_t K) {
  return (int64_t)split_k(M, Nn, K).n * M * Nn;
}

// Sum segment of per-block column-sum partials [blocks][cols] into out[cols].
tri::SumSeg colsum_segment(const float *part, int64_t cols, float *out) {
  return tri::SumSeg{part, tri::proj_partials(), cols, cols, out, cols, cols};
}

}  // namespace

extern "C" {

tri_attn_status tri_proj_workspace_size(const tri_proj_problem *prob, size_t *bytes) {
  tri_attn_status st = check_proj(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!bytes) return TRI_ATTN_ERR_INVALID_ARG;
  *bytes = carve_proj(prob, nullptr, nullptr);
  return TRI_ATTN_OK;
}

tri_attn_status tri_proj_in_fwd(const tri_proj_problem *prob, const void *z, const float *gamma,
                                const float *beta, const void *w_qkvg, const float *b_g,
                                const void *w_b, void *x, float *stats, void *q, void *k,
                                void *v, void *g, void *bias, void *workspace,
                                size_t workspace_bytes, tri_attn_stream_t stream_) {
  ProjWs ws;
  tri_attn_status st = proj_begin(prob, workspace, workspace_bytes, &ws);
  if (st != TRI_ATTN_OK) return st;
  for (const void *p : {(const void *)gamma, (const void *)beta, w_qkvg, (const void *)b_g, w_b})
    TRI_CHECK_PTR(p);
  const int64_t R = proj_total_rows(prob), cz = prob->cz, hc = (int64_t)prob->H * prob->c;
  if (R == 0) return TRI_ATTN_OK;      // no rows: nothing to do, nothing enqueued
  for (const void *p : {z, (const void *)x, (const void *)stats, (const void *)q, (const void *)k,
                        (const void *)v, (const void *)g, (const void *)bias})
    TRI_CHECK_PTR(p);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaMemsetAsync(ws.status, 0, sizeof(int32_t), stream) != cudaSuccess)
    return TRI_ATTN_ERR_CUDA;
  tri::ProjArgs a{};
  a.rows = R;
  a.rows_per = prob->rows;
  a.cz = prob->cz;
  a.H = prob->H;
  a.eps = prob->eps;
  a.z = static_cast<const __nv_bfloat16 *>(z);
  a.gamma = gamma;
  a.beta = beta;
  a.w_b = static_cast<const __nv_bfloat16 *>(w_b);
  a.x = static_cast<__nv_bfloat16 *>(x);
  a.stats = stats;
  a.bias = static_cast<__nv_bfloat16 *>(bias);
  st = cuda_status(tri::launch_ln_fwd(a, stream));
  if (st != TRI_ATTN_OK) return st;
  // q | k | v | g = x w_qkvg: x K-major, w_qkvg [cz][4Hc] MN-major, each
  // 64-column box of the product routed to its output, b_g added to g
  tri::GemmMaps ys;
  tri::GemmMaps xs;
  tri::GemmOuts outs;
  void *dst[4] = {q, k, v, g};
  if (!encode_operand(&xs.map[0], x, false, R, cz, 1) ||
      !encode_operand(&ys.map[0], w_qkvg, true, 4 * hc, cz, 1))
    return TRI_ATTN_ERR_CUDA;
  for (int o = 0; o < 4; ++o)
    if (!encode_stack(&outs.map[o], dst[o], false, hc, R, 1, 64, 32)) return TRI_ATTN_ERR_CUDA;
  tri::GemmArgs args{};
  args.M = (int)R;
  args.Nn = (int)(4 * hc);
  args.K = (int)cz;
  args.batch = 1;
  args.nouts = 4;
  args.cols_per_out = (int)hc;
  args.k_per_x = 1 << 30;
  args.col_bias = b_g;
  args.col_bias_from = (int)(3 * hc);
  args.status = ws.status;
  return cuda_status(tri::launch_gemm_tc(false, true, false, xs, ys, outs, args, stream));
}

tri_attn_status tri_proj_in_bwd(const tri_proj_problem *prob, const void *z, const float *gamma,
                                const void *w_qkvg, const void *w_b, const void *x,
                                const float *stats, const void *dq, const void *dk,
                                const void *dv, const void *dg, const void *dbias, void *dz,
                                float *dgamma, float *dbeta, float *dw_qkvg, float *db_g,
                                float *dw_b, void *workspace, size_t workspace_bytes,
                                tri_attn_stream_t stream_) {
  ProjWs ws;
  tri_attn_status st = proj_begin(prob, workspace, workspace_bytes, &ws);
  if (st != TRI_ATTN_OK) return st;
  for (const void *p : {(const void *)gamma, w_qkvg, w_b, (const void *)dgamma,
                        (const void *)dbeta, (const void *)dw_qkvg, (const void *)db_g,
                        (const void *)dw_b})
    TRI_CHECK_PTR(p);
  const int64_t R = proj_total_rows(prob), cz = prob->cz, hc = (int64_t)prob->H * prob->c;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (R == 0) {
    // no rows: every parameter gradient is an empty sum
    for (auto t : {std::make_pair(dgamma, cz), std::make_pair(dbeta, cz),
                   std::make_pair(dw_qkvg, cz * 4 * hc), std::make_pair(db_g, hc),
                   std::make_pair(dw_b, cz * prob->H)})
      if ((st = zero_f32(t.first, (size_t)t.second, stream)) != TRI_ATTN_OK) return st;
    return TRI_ATTN_OK;
  }
  for (const void *p : {z, x, (const void *)stats, dq, dk, dv, dg, dbias, (const void *)dz})
    TRI_CHECK_PTR(p);
  if (cudaMemsetAsync(ws.status, 0, sizeof(int32_t), stream) != cudaSuccess)
    return TRI_ATTN_ERR_CUDA;
  // dx = [dq dk dv dg] w_qkvg^T (fp32): four K-major X maps along K, w_qkvg K-major
  {
    tri::GemmMaps ys;
    tri::GemmMaps xs;
    tri::GemmOuts outs;
    const void *src[4] = {dq, dk, dv, dg};
    for (int o = 0; o < 4; ++o)
      if (!encode_operand(&xs.map[o], src[o], false, R, hc, 1)) return TRI_ATTN_ERR_CUDA;
    if (!encode_operand(&ys.map[0], w_qkvg, false, cz, 4 * hc, 1) ||
        !encode_stack(&outs.map[0], ws.dx, true, cz, R, 1, 32, 32))
      return TRI_ATTN_ERR_CUDA;
    tri::GemmArgs args{};
    args.M = (int)R;
    args.Nn = (int)cz;
    args.K = (int)(4 * hc);
    args.batch = 1;
    args.nouts = 1;
    args.cols_per_out = (int)cz;
    args.k_per_x = (int)hc;
    args.status = ws.status;
    st = cuda_status(tri::launch_gemm_tc(false, false, true, xs, ys, outs, args, stream));
    if (st != TRI_ATTN_OK) return st;
  }
  // LayerNorm backward: dz, and per-warp partials of dgamma | dbeta | dw_b
  tri::ProjArgs a{};
  a.rows = R;
  a.rows_per = prob->rows;
  a.cz = prob->cz;
  a.H = prob->H;
  a.eps = prob->eps;
  a.z = static_cast<const __nv_bfloat16 *>(z);
  a.gamma = gamma;
  a.w_b = static_cast<const __nv_bfloat16 *>(w_b);
  a.x = static_cast<__nv_bfloat16 *>(const_cast<void *>(x));
  a.stats = const_cast<float *>(stats);
  a.dx = ws.dx;
  a.dbias = static_cast<const __nv_bfloat16 *>(dbias);
  a.dz = static_cast<__nv_bfloat16 *>(dz);
  a.part = ws.part;
  a.status = ws.status;
  cudaError_t e = tri::launch_ln_bwd(a, stream);
  // the db_g column-sum partials follow the LayerNorm partials; one launch sums both
  const int64_t warps = tri::proj_partials(), pw = cz * (2 + prob->H);
  float *cpart = ws.part + warps * pw;
  if (e == cudaSuccess)
    e = tri::launch_colsum(static_cast<const __nv_bfloat16 *>(dg), R, (int)hc, cpart, stream);
  if (e == cudaSuccess) {
    const tri::SumSeg segs[4] = {
        {ws.part, warps, pw, cz, dgamma, cz, cz},
        {ws.part + cz, warps, pw, cz, dbeta, cz, cz},
        {ws.part + 2 * cz, warps, pw, cz * prob->H, dw_b, cz * prob->H, cz * prob->H},
        colsum_segment(cpart, hc, db_g)};
    e = tri::launch_ordered_sums(segs, 4, stream);
  }
  if ((st = cuda_status(e)) != TRI_ATTN_OK) return st;
  // dw_qkvg = x^T [dq dk dv dg]
  const void *grads[4] = {dq, dk, dv, dg};
  return weight_grad(x, grads, 4, cz, 4 * hc, R, dw_qkvg, ws, stream);
}

tri_attn_status tri_proj_out_fwd(const tri_proj_problem *prob, const void *o, const void *w_o,
                                 const float *b_o, void *y, void *workspace,
                                 size_t workspace_bytes, tri_attn_stream_t stream_) {
  ProjWs ws;
  tri_attn_status st = proj_begin(prob, workspace, workspace_bytes, &ws);
  if (st != TRI_ATTN_OK) return st;
  for (const void *p : {w_o, (const void *)b_o}) TRI_CHECK_PTR(p);
  const int64_t R = proj_total_rows(prob), cz = prob->cz, hc = (int64_t)prob->H * prob->c;
  if (R == 0) return TRI_ATTN_OK;      // no rows: nothing to do, nothing enqueued
  for (const void *p : {o, (const void *)y}) TRI_CHECK_PTR(p);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaMemsetAsync(ws.status, 0, sizeof(int32_t), stream) != cudaSuccess)
    return TRI_ATTN_ERR_CUDA;
  // y = o w_o + b_o: o K-major, w_o [Hc][cz] MN-major
  tri::GemmMaps ys;
  tri::GemmMaps xs;
  tri::GemmOuts outs;
  if (!encode_operand(&xs.map[0], o, false, R, hc, 1) ||
      !encode_operand(&ys.map[0], w_o, true, cz, hc, 1) ||
      !encode_stack(&outs.map[0], y, false, cz, R, 1, 64, 32))
    return TRI_ATTN_ERR_CUDA;
  tri::GemmArgs args{};
  args.M = (int)R;
  args.Nn = (int)cz;
  args.K = (int)hc;
  args.batch = 1;
  args.nouts = 1;
  args.cols_per_out = (int)cz;
  args.k_per_x = 1 << 30;
  args.col_bias = b_o;
  args.col_bias_from = 0;
  args.status = ws.status;
  return cuda_status(tri::launch_gemm_tc(false, true, false, xs, ys, outs, args, stream));
}

tri_attn_status tri_proj_out_bwd(const tri_proj_problem *prob, const void *o, const void *w_o,
                                 const void *dy, void *do_, float *dw_o, float *db_o,
                                 void *workspace, size_t workspace_bytes,
                                 tri_attn_stream_t stream_) {
  ProjWs ws;
  tri_attn_status st = proj_begin(prob, workspace, workspace_bytes, &ws);
  if (st != TRI_ATTN_OK) return st;
  for (const void *p : {w_o, (const void *)dw_o, (const void *)db_o}) TRI_CHECK_PTR(p);
  const int64_t R = proj_total_rows(prob), cz = prob->cz, hc = (int64_t)prob->H * prob->c;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (R == 0) {
    if ((st = zero_f32(dw_o, (size_t)(hc * cz), stream)) != TRI_ATTN_OK) return st;
    return zero_f32(db_o, (size_t)cz, stream);
  }
  for (const void *p : {o, dy, (const void *)do_}) TRI_CHECK_PTR(p);
  if (cudaMemsetAsync(ws.status, 0, sizeof(int32_t), stream) != cudaSuccess)
    return TRI_ATTN_ERR_CUDA;
  // do = dy w_o^T: dy K-major, w_o [Hc][cz] K-major
  {
    tri::GemmMaps ys;
    tri::GemmMaps xs;
    tri::GemmOuts outs;
    if (!encode_operand(&xs.map[0], dy, false, R, cz, 1) ||
        !encode_operand(&ys.map[0], w_o, false, hc, cz, 1) ||
        !encode_stack(&outs.map[0], do_, false, hc, R, 1, 64, 32))
      return TRI_ATTN_ERR_CUDA;
    tri::GemmArgs args{};
    args.M = (int)R;
    args.Nn = (int)hc;
    args.K = (int)cz;
    args.batch = 1;
    args.nouts = 1;
    args.cols_per_out = (int)hc;
    args.k_per_x = 1 << 30;
    args.status = ws.status;
    st = cuda_status(tri::launch_gemm_tc(false, false, false, xs, ys, outs, args, stream));
    if (st != TRI_ATTN_OK) return st;
  }
  // dW_o split-K partials, then the db_o column-sum partials after them; one sum launch
  tri::SumSeg segs[2];
  if ((st = weight_grad(o, &dy, 1, hc, cz, R, dw_o, ws, stream, &segs[0])) != TRI_ATTN_OK)
    return st;
  float *cpart = ws.part + weight_grad_partials(hc, cz, R);
  cudaError_t e = tri::launch_colsum(static_cast<const __nv_bfloat16 *>(dy), R, (int)cz, cpart,
                                     stream);
  if (e != cudaSuccess) return cuda_status(e);
  segs[1] = colsum_segment(cpart, cz, db_o);
  return cuda_status(tri::launch_ordered_sums(segs, 2, stream));
}

// ----------------------------------------- triangle multiplicative update --

namespace {

struct MulUpdSaved {
  __nv_bfloat16 *x, *pg, *a_cm, *b_cm, *t_pm, *u, *h;
  float *stats, *stats_o;
};

struct MulUpdWs {
  int32_t *status;
  __nv_bfloat16 *zero_wb, *zero_bias, *bias_scratch;   // the LayerNorm kernels' bias head
  __nv_bfloat16 *t_cm;                                 // forward
  __nv_bfloat16 *dh, *dpg, *dt_pm, *dt_cm, *da_cm, *db_cm;   // backward
  float *du, *dx, *part;
};

tri_attn_status check_mul_update(const tri_mul_update_problem *p) {
  if (!p) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->N < 0 || p->N > kMaxN || !(p->eps > 0.0f)) return TRI_ATTN_ERR_INVALID_ARG;
  if (p->direction != TRI_MUL_OUTGOING && p->direction != TRI_MUL_INCOMING)
    return TRI_ATTN_ERR_INVALID_ARG;
  auto channels_ok = [](int v) { return v == 64 || v == 128 || v == 192 || v == 256; };
  if (!channels_ok(p->cz) || !channels_ok(p->c) || p->N % 8 != 0)
    return TRI_ATTN_ERR_UNSUPPORTED;
  return TRI_ATTN_OK;
}

size_t carve_mul_update_saved(const tri_mul_update_problem *p, void *base, MulUpdSaved *out) {
  Carver c(base);
  MulUpdSaved s{};
  const size_t R = (size_t)p->N * p->N, cz = p->cz, ch = p->c, pgw = 4 * ch + cz;
  s.x = static_cast<__nv_bfloat16 *>(c.take(2 * R * cz));
  s.stats = static_cast<float *>(c.take(8 * R));
  s.pg = static_cast<__nv_bfloat16 *>(c.take(2 * R * pgw));
  s.a_cm = static_cast<__nv_bfloat16 *>(c.take(2 * R * ch));
  s.b_cm = static_cast<__nv_bfloat16 *>(c.take(2 * R * ch));
  s.t_pm = static_cast<__nv_bfloat16 *>(c.take(2 * R * ch));
  s.u = static_cast<__nv_bfloat16 *>(c.take(2 * R * ch));
  s.stats_o = static_cast<float *>(c.take(8 * R));
  s.h = static_cast<__nv_bfloat16 *>(c.take(2 * R * cz));
  if (out) *out = s;
  return c.off;
}

// A common head (status word, the zero bias head of the LayerNorm kernels),
// then the forward's buffers and the backward's sharing one region.
size_t carve_mul_update_ws(const tri_mul_update_problem *p, void *base, MulUpdWs *out) {
  Carver c(base);
  MulUpdWs w{};
  const int64_t R = p->N * p->N, cz = p->cz, ch = p->c, pgw = 4 * ch + cz;
  w.status = static_cast<int32_t *>(c.take(sizeof(int32_t)));
  w.zero_wb = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)std::max(cz, ch)));
  w.zero_bias = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)R));
  w.bias_scratch = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)R));
  const size_t head = c.off;
  // forward
  w.t_cm = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)(R * ch)));
  const size_t fwd_end = c.off;
  // backward, from the same offset
  c.off = head;
  w.dh = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)(R * cz)));
  w.dpg = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)(R * pgw)));
  w.dt_pm = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)(R * ch)));
  w.dt_cm = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)(R * ch)));
  w.da_cm = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)(R * ch)));
  w.db_cm = static_cast<__nv_bfloat16 *>(c.take(2 * (size_t)(R * ch)));
  w.du = static_cast<float *>(c.take(4 * (size_t)(R * ch)));
  w.dx = static_cast<float *>(c.take(4 * (size_t)(R * cz)));
  const int64_t blocks = tri::proj_partials();
  int64_t part = std::max<int64_t>(blocks * 3 * std::max(cz, ch), blocks * pgw);
  if (R > 0) {
    part = std::max(part, weight_grad_partials(cz, pgw, R));
    part = std::max(part, weight_grad_partials(ch, cz, R));
  }
  w.part = static_cast<float *>(c.take(4 * (size_t)part));
  if (out) *out = w;
  return std::max(fwd_end, c.off);
}

// One LayerNorm over `ch` channels through the projection kernels, with a
// single bias head of zeros whose output is discarded.
tri::ProjArgs ln_args(const MulUpdWs &w, int64_t R, int ch, float eps, const void *z,
                      const float *gamma, const float *beta, __nv_bfloat16 *x, float *stats) {
  tri::ProjArgs a{};
  a.rows = R;
  a.rows_per = R;
  a.cz = ch;
  a.H = 1;
  a.eps = eps;
  a.z = static_cast<const __nv_bfloat16 *>(z);
  a.gamma = gamma;
  a.beta = beta;
  a.w_b = w.zero_wb;
  a.x = x;
  a.stats = stats;
  a.bias = w.bias_scratch;
  a.dbias = w.zero_bias;
  a.part = w.part;
  a.status = w.status;
  return a;
}

// D [M][Nn] = X Y^T with X [M][K] K-major and Y as stored (MN-major [K][Nn] or
// K-major [Nn][K]); bf16 output with an optional column bias, or fp32.
tri_attn_status product(const void *x, const void *y, bool y_mn, void *out, bool f32, int64_t M,
                        int64_t Nn, int64_t K, const float *bias, int32_t *status,
                        cudaStream_t stream) {
  tri::GemmMaps xs, ys;
  tri::GemmOuts outs;
  if (!encode_operand(&xs.map[0], x, false, M, K, 1) ||
      !encode_operand(&ys.map[0], y, y_mn, Nn, K, 1) ||
      !encode_stack(&outs.map[0], out, f32, Nn, M, 1, f32 ? 32 : 64, 32))
    return TRI_ATTN_ERR_CUDA;
  tri::GemmArgs args{};
  args.M = (int)M;
  args.Nn = (int)Nn;
  args.K = (int)K;
  args.batch = 1;
  args.nouts = 1;
  args.cols_per_out = (int)Nn;
  args.k_per_x = 1 << 30;
  args.col_bias = bias;
  args.col_bias_from = 0;
  args.status = status;
  return cuda_status(tri::launch_gemm_tc(false, y_mn, f32, xs, ys, outs, args, stream));
}

tri_attn_status mul_update_begin(const tri_mul_update_problem *p,
                                 const tri_mul_update_params *w, const void *saved,
                                 size_t saved_bytes, void *ws, size_t ws_bytes) {
  tri_attn_status st = check_mul_update(p);
  if (st != TRI_ATTN_OK) return st;
  if (!w) return TRI_ATTN_ERR_INVALID_ARG;
  for (const void *q : {(const void *)w->ln_gamma, (const void *)w->ln_beta, w->w_in,
                        (const void *)w->b_in, (const void *)w->ln_out_gamma,
                        (const void *)w->ln_out_beta, w->w_o, (const void *)w->b_o})
    TRI_CHECK_PTR(q);
  if (!ws || !aligned16(ws) || ws_bytes < carve_mul_update_ws(p, nullptr, nullptr))
    return TRI_ATTN_ERR_WORKSPACE;
  if (!saved || !aligned16(saved) || saved_bytes < carve_mul_update_saved(p, nullptr, nullptr))
    return TRI_ATTN_ERR_WORKSPACE;
  return TRI_ATTN_OK;
}

}  // namespace

tri_attn_status tri_mul_update_sizes(const tri_mul_update_problem *prob, size_t *saved_bytes,
                                     size_t *workspace_bytes) {
  tri_attn_status st = check_mul_update(prob);
  if (st != TRI_ATTN_OK) return st;
  if (!saved_bytes || !workspace_bytes) return TRI_ATTN_ERR_INVALID_ARG;
  *saved_bytes = carve_mul_update_saved(prob, nullptr, nullptr);
  *workspace_bytes = carve_mul_update_ws(prob, nullptr, nullptr);
  return TRI_ATTN_OK;
}

tri_attn_status tri_mul_update_fwd(const tri_mul_update_problem *prob,
                                   const tri_mul_update_params *params, const void *z, void *y,
                                   void *saved, size_t saved_bytes, void *workspace,
                                   size_t workspace_bytes, tri_attn_stream_t stream_) {
  tri_attn_status st =
      mul_update_begin(prob, params, saved, saved_bytes, workspace, workspace_bytes);
  if (st != TRI_ATTN_OK) return st;
  if (prob->N == 0) return TRI_ATTN_OK;
  TRI_CHECK_PTR(z);
  TRI_CHECK_PTR(y);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  MulUpdSaved s;
  MulUpdWs w;
  carve_mul_update_saved(prob, saved, &s);
  carve_mul_update_ws(prob, workspace, &w);
  const int64_t R = prob->N * prob->N, cz = prob->cz, ch = prob->c, pgw = 4 * ch + cz;
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(int32_t), stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(w.zero_wb, 0, 2 * (size_t)std::max(cz, ch), stream);
  if (e != cudaSuccess) return cuda_status(e);
  // x = LayerNorm(z)
  tri::ProjArgs a = ln_args(w, R, (int)cz, prob->eps, z, params->ln_gamma, params->ln_beta,
                            s.x, s.stats);
  if ((st = cuda_status(tri::launch_ln_fwd(a, stream))) != TRI_ATTN_OK) return st;
  // [ap | ag | bp | bg | gl] = x W_in + b_in
  if ((st = product(s.x, params->w_in, true, s.pg, false, R, pgw, cz, params->b_in, w.status,
                    stream)) != TRI_ATTN_OK)
    return st;
  // a, b channel-major; t = their contraction (channel-major), then pair-major
  if ((st = cuda_status(tri::launch_gate_in_fwd(s.pg, R, (int)ch, pgw, s.a_cm, s.b_cm,
                                                stream))) != TRI_ATTN_OK)
    return st;
  const tri_mul_problem mp{prob->N, (int32_t)ch, prob->direction};
  const bool mn = prob->direction == TRI_MUL_INCOMING;
  if ((st = mul_product(&mp, s.a_cm, mn, s.b_cm, mn, w.t_cm, w.status, stream)) != TRI_ATTN_OK)
    return st;
  if ((st = cuda_status(tri::launch_transpose(w.t_cm, ch, R, s.t_pm, stream))) != TRI_ATTN_OK)
    return st;
  // u = LayerNorm_out(t); h = u W_o + b_o; y = sigmoid(gl) h
  a = ln_args(w, R, (int)ch, prob->eps, s.t_pm, params->ln_out_gamma, params->ln_out_beta, s.u,
              s.stats_o);
  if ((st = cuda_status(tri::launch_ln_fwd(a, stream))) != TRI_ATTN_OK) return st;
  if ((st = product(s.u, params->w_o, true, s.h, false, R, cz, ch, params->b_o, w.status,
                    stream)) != TRI_ATTN_OK)
    return st;
  return cuda_status(tri::launch_out_fwd(s.pg, pgw, (int)(4 * ch), s.h, R, (int)cz,
                                         static_cast<__nv_bfloat16 *>(y), stream));
}

tri_attn_status tri_mul_update_bwd(const tri_mul_update_problem *prob,
                                   const tri_mul_update_params *params, const void *z,
                                   const void *saved, size_t saved_bytes, const void *dy,
                                   void *dz, const tri_mul_update_grads *grads, void *workspace,
                                   size_t workspace_bytes, tri_attn_stream_t stream_) {
  tri_attn_status st =
      mul_update_begin(prob, params, saved, saved_bytes, workspace, workspace_bytes);
  if (st != TRI_ATTN_OK) return st;
  if (!grads) return TRI_ATTN_ERR_INVALID_ARG;
  for (const void *q : {(const void *)grads->ln_gamma, (const void *)grads->ln_beta,
                        (const void *)grads->w_in, (const void *)grads->b_in,
                        (const void *)grads->ln_out_gamma, (const void *)grads->ln_out_beta,
                        (const void *)grads->w_o, (const void *)grads->b_o})
    TRI_CHECK_PTR(q);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int64_t R = prob->N * prob->N, cz = prob->cz, ch = prob->c, pgw = 4 * ch + cz;
  if (R == 0) {
    // no pair positions: every parameter gradient is an empty sum
    for (auto t : {std::make_pair(grads->ln_gamma, cz), std::make_pair(grads->ln_beta, cz),
                   std::make_pair(grads->w_in, cz * pgw), std::make_pair(grads->b_in, pgw),
                   std::make_pair(grads->ln_out_gamma, ch), std::make_pair(grads->ln_out_beta, ch),
                   std::make_pair(grads->w_o, ch * cz), std::make_pair(grads->b_o, cz)})
      if ((st = zero_f32(t.first, (size_t)t.second, stream)) != TRI_ATTN_OK) return st;
    return TRI_ATTN_OK;
  }
  TRI_CHECK_PTR(z);
  TRI_CHECK_PTR(dy);
  TRI_CHECK_PTR(dz);
  MulUpdSaved s;
  MulUpdWs w;
  carve_mul_update_saved(prob, const_cast<void *>(saved), &s);
  carve_mul_update_ws(prob, workspace, &w);
  const ProjWs pw{w.status, w.dx, w.part};
  const int64_t blocks = tri::proj_partials();
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(int32_t), stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(w.zero_wb, 0, 2 * (size_t)std::max(cz, ch), stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(w.zero_bias, 0, 2 * (size_t)R, stream);
  if (e != cudaSuccess) return cuda_status(e);
  // dh = dy sigmoid(gl); dgl into the last cz columns of dpg
  if ((st = cuda_status(tri::launch_out_bwd(static_cast<const __nv_bfloat16 *>(dy), s.pg, pgw,
                                            (int)(4 * ch), s.h, R, (int)cz, w.dh, w.dpg,
                                            stream))) != TRI_ATTN_OK)
    return st;
  // dW_o = u^T dh, db_o = column sums of dh, du = dh W_o^T (fp32)
  const void *dh_list[1] = {w.dh};
  if ((st = weight_grad(s.u, dh_list, 1, ch, cz, R, grads->w_o, pw, stream)) != TRI_ATTN_OK)
    return st;
  e = tri::launch_colsum(w.dh, R, (int)cz, w.part, stream);
  if (e == cudaSuccess) {
    const tri::SumSeg seg = colsum_segment(w.part, cz, grads->b_o);
    e = tri::launch_ordered_sums(&seg, 1, stream);
  }
  if ((st = cuda_status(e)) != TRI_ATTN_OK) return st;
  if ((st = product(w.dh, params->w_o, false, w.du, true, R, ch, cz, nullptr, w.status,
                    stream)) != TRI_ATTN_OK)
    return st;
  // LayerNorm_out backward: dt (pair-major), dgamma_o, dbeta_o
  tri::ProjArgs a = ln_args(w, R, (int)ch, prob->eps, s.t_pm, params->ln_out_gamma, nullptr,
                            s.u, s.stats_o);
  a.dx = w.du;
  a.dz = w.dt_pm;
  e = tri::launch_ln_bwd(a, stream);
  if (e == cudaSuccess) {
    const tri::SumSeg segs[2] = {{w.part, blocks, 3 * ch, ch, grads->ln_out_gamma, ch, ch},
                                 {w.part + ch, blocks, 3 * ch, ch, grads->ln_out_beta, ch, ch}};
    e = tri::launch_ordered_sums(segs, 2, stream);
  }
  if (e == cudaSuccess) e = tri::launch_transpose(w.dt_pm, R, ch, w.dt_cm, stream);
  if ((st = cuda_status(e)) != TRI_ATTN_OK) return st;
  // the contraction's backward (as tri_mul_bwd), then the gates': dpg columns 0 .. 4c
  const tri_mul_problem mp{prob->N, (int32_t)ch, prob->direction};
  if (prob->direction == TRI_MUL_OUTGOING) {
    st = mul_product(&mp, w.dt_cm, false, s.b_cm, true, w.da_cm, w.status, stream);
    if (st == TRI_ATTN_OK)
      st = mul_product(&mp, w.dt_cm, true, s.a_cm, true, w.db_cm, w.status, stream);
  } else {
    st = mul_product(&mp, s.b_cm, false, w.dt_cm, false, w.da_cm, w.status, stream);
    if (st == TRI_ATTN_OK)
      st = mul_product(&mp, s.a_cm, false, w.dt_cm, true, w.db_cm, w.status, stream);
  }
  if (st != TRI_ATTN_OK) return st;
  if ((st = cuda_status(tri::launch_gate_in_bwd(w.da_cm, w.db_cm, s.pg, R, (int)ch, pgw, w.dpg,
                                                stream))) != TRI_ATTN_OK)
    return st;
  // db_in = column sums of dpg; dW_in = x^T dpg; dx = dpg W_in^T (fp32)
  e = tri::launch_colsum_strided(w.dpg, R, pgw, (int)pgw, w.part, stream);
  if (e == cudaSuccess) {
    const tri::SumSeg seg = colsum_segment(w.part, pgw, grads->b_in);
    e = tri::launch_ordered_sums(&seg, 1, stream);
  }
  if ((st = cuda_status(e)) != TRI_ATTN_OK) return st;
  const void *dpg_list[1] = {w.dpg};
  if ((st = weight_grad(s.x, dpg_list, 1, cz, pgw, R, grads->w_in, pw, stream)) != TRI_ATTN_OK)
    return st;
  if ((st = product(w.dpg, params->w_in, false, w.dx, true, R, cz, pgw, nullptr, w.status,
                    stream)) != TRI_ATTN_OK)
    return st;
  // LayerNorm backward: dz, dgamma, dbeta
  a = ln_args(w, R, (int)cz, prob->eps, z, params->ln_gamma, nullptr, s.x, s.stats);
  a.dx = w.dx;
  a.dz = static_cast<__nv_bfloat16 *>(dz);
  e = tri::launch_ln_bwd(a, stream);
  if (e == cudaSuccess) {
    const tri::SumSeg segs[2] = {{w.part, blocks, 3 * cz, cz, grads->ln_gamma, cz, cz},
                                 {w.part + cz, blocks, 3 * cz, cz, grads->ln_beta, cz, cz}};
    e = tri::launch_ordered_sums(segs, 2, stream);
  }
  return cuda_status(e);
}

}  // extern "C"
