// cta_certified_topk_attn_noalloc: the certified Top-k call for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: code running while a CUDA graph is
// being captured on a stream where allocation is not allowed, plugins of
// inference runtimes that forbid device allocation outside their own pool,
// and callers with a hard device-memory budget fixed at start-up.  They
// cannot provide the caller-owned workspace that cta_certified_topk_attn
// needs, so this entry point supplies it from a fixed array compiled into the
// library instead.
//
// The scratch is a file-scope __device__ array of CTA_NOALLOC_SCRATCH_BYTES.
// In host code its name is only a host-side stand-in; the device address is
// obtained with cudaGetSymbolAddress, once per device, on the first call made
// while that device is current, and cached.  That first call should therefore
// happen before any stream capture.  Nothing here allocates: no cudaMalloc,
// no cudaFree, no allocating library routine.
#include <cuda_runtime.h>

#include <mutex>

#include "cta.h"

namespace {

constexpr size_t kScratchBytes = CTA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 128;

// Shared by every call on a device; it keeps the last call's contents.  Every
// region the kernels read is written earlier in the same call, so nothing has
// to be cleared between calls.
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

int scratch_address(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CTA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return CTA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return CTA_OK;
}

}  // namespace

extern "C" int cta_certified_topk_attn_noalloc(const void* q, const void* K, const void* V,
                                               int64_t n, int d, int n_heads, int n_kv_heads,
                                               double eps, void* out, int32_t* k_out,
                                               int32_t* idx_out, float* tv_out,
                                               const cta_opts* opts) {
  cta_opts o;
  if (opts) o = *opts;
  else cta_opts_init(&o);
  const size_t need = cta_workspace_size(n, d, n_heads, n_kv_heads, &o);
  if (need == 0) return CTA_ERR_SHAPE;
  if (need > kScratchBytes) return CTA_ERR_TOO_LARGE;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != CTA_OK) return rc;
  o.workspace = scratch;
  o.workspace_bytes = kScratchBytes;
  return cta_certified_topk_attn(q, K, V, n, d, n_heads, n_kv_heads, eps, out, k_out, idx_out,
                                 tv_out, &o);
}
