// tri_attn_fwd_noalloc: the forward with its scratch in a file-scope device
// array instead of a caller-provided workspace (see include/tri_attn.h).
#include <cstddef>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/tri_attn.h"

namespace {

constexpr size_t kScratchBytes = TRI_ATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 128;

// One copy per GPU that loads the library. In host code this name is only a
// stand-in for the symbol: its device address comes from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device with that device current.
tri_attn_status scratch_on_current_device(void **ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return TRI_ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
      return TRI_ATTN_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
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
  st = scratch_on_current_device(&scratch);
  if (st != TRI_ATTN_OK) return st;
  return tri_attn_fwd(prob, q, k, v, bias, gate, mask, out, lse, scratch, kScratchBytes, stream);
}
