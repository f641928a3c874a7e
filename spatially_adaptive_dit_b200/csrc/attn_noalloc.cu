// The tail-balanced attention (safedit_attn_subset_ws) with its workspace
// taken from a fixed device array of this library instead of the caller, for
// callers that may not allocate device memory around the call.  The pages
// have no counterpart: SAFE-DiT defines the SRSU rows (방법론 3), not where a
// launch keeps its partial results.
//
// The array is kAttnScratchBytes per device, reserved when the library's
// device code is loaded on that device.  Its address is looked up once per
// device (cudaGetSymbolAddress, on the first call with that device current)
// and cached; nothing is allocated afterwards.  The partial results are
// written in full before the merge reads them, so nothing in the array has
// to start at zero and nothing is cleared.  All calls on one device share the
// array: calls that overlap on the GPU (other streams, other host threads)
// race on it.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "safedit.h"

namespace {

constexpr size_t kAttnScratchBytes = SAFEDIT_ATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_attn_scratch[kAttnScratchBytes];

std::atomic<void*> g_scratch_addr[kMaxDevices];

// The array's address on the current device, looked up on first use.
safedit_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAFEDIT_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SAFEDIT_ERR_UNSUPPORTED;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || p == nullptr) return SAFEDIT_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return SAFEDIT_OK;
}

}  // namespace

extern "C" safedit_status safedit_attn_subset_noalloc(const safedit_tensor* q, const safedit_tensor* k,
                                                      const safedit_tensor* v, const int32_t* d_idx,
                                                      int32_t n_idx, const safedit_tensor* key_pad,
                                                      const safedit_tensor* bias, float scale,
                                                      const safedit_tensor* out, int32_t out_scattered,
                                                      void* stream) {
  if (!q || !k || q->ndim != 4 || k->ndim != 4) return SAFEDIT_ERR_INVALID_ARG;
  const int64_t n_rows = d_idx ? int64_t(n_idx) : q->dims[2];
  const size_t need = safedit_attn_subset_workspace_size(q->dims[0], q->dims[1], n_rows, k->dims[2],
                                                         int32_t(q->dims[3]));
  if (need > kAttnScratchBytes) return SAFEDIT_ERR_UNSUPPORTED;  // before any launch
  void* scratch = nullptr;
  const safedit_status st = scratch_address(&scratch);
  if (st != SAFEDIT_OK) return st;
  return safedit_attn_subset_ws(q, k, v, d_idx, n_idx, key_pad, bias, scale, out, out_scattered, scratch,
                                kAttnScratchBytes, stream);
}
