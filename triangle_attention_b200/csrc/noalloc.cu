// tri_attn_fwd_noalloc: the forward with its scratch in a file-scope device
// array instead of a caller-provided workspace (see include/tri_attn.h).
#include <cstddef>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/tri_attn.h"

namespace {

constexpr size_t kScratchBytes = TRI_ATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 128;

// One copy per GPU that loads the library. In host code this name is only a
// stand-in for the symbol: its device address comes from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Driver entry points, resolved through the runtime (libcuda is not linked).
template <typename Fn>
Fn driver_fn(const char *name) {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

struct Cached {
  unsigned long long ctx_id;   // unique id of the context the address belongs to
  void *ptr;
};

std::mutex g_mu;
Cached g_cache[kMaxDevices];

// Device address of the scratch array in the current context. The address is
// looked up with the device current and kept per device together with the
// context's unique id; a different context on that device (after
// cudaDeviceReset, or a context the caller made current) looks it up again.
tri_attn_status scratch_in_current_context(void **ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return TRI_ATTN_ERR_CUDA;
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return TRI_ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return TRI_ATTN_ERR_CUDA;
  void *p = nullptr;
  if (!ctx) {
    // no context yet: the symbol lookup makes the runtime create the device's
    // primary context, which is then current
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p ||
        get_current(&ctx) != CUDA_SUCCESS || !ctx)
      return TRI_ATTN_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return TRI_ATTN_ERR_CUDA;
  Cached &c = g_cache[dev];
  if (!c.ptr || c.ctx_id != id) {
    if (!p && (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p))
      return TRI_ATTN_ERR_CUDA;
    c.ptr = p;
    c.ctx_id = id;
  }
  *ptr = c.ptr;
  return TRI_ATTN_OK;
}

}  // namespace

extern "C" tri_attn_status tri_attn_fwd_noalloc(const tri_attn_problem *prob, const void *q,
                                                const void *k, const void *v, const void *bias,
                                                const void *gate, const uint8_t *mask, void *out,
                                                float *lse, tri_attn_stream_t stream) {
  size_t need = 0;
  tri_attn_status st = tri_attn_fwd_workspace_size(prob, &need);
  if (st != TRI_ATTN_OK) return st;
  if (need > kScratchBytes) return TRI_ATTN_ERR_WORKSPACE;
  void *scratch = nullptr;
  st = scratch_in_current_context(&scratch);
  if (st != TRI_ATTN_OK) return st;
  return tri_attn_fwd(prob, q, k, v, bias, gate, mask, out, lse, scratch, kScratchBytes, stream);
}
