// host.cu -- library-wide host state of libsafedit.so: the per-device status
// word, status strings, the kernel launch counter, the debug wait limit and
// the TMA descriptor encoder.
#include <atomic>
#include <mutex>
#include <unordered_map>

#include <cudaTypedefs.h>

#include "internal.h"

// One status word per device: the first device-detected error since the last
// safedit_get_device_status(), and the word that call takes out of it.
// Static storage: the library allocates nothing.
static __device__ int g_device_status;
static __device__ int g_status_taken;

// Reads and clears the status word in one atomic step, so that an error a
// kernel on another stream records at the same moment is either returned
// now or kept for the next read, never lost.
__global__ void status_take_kernel() { g_status_taken = atomicExch(&g_device_status, 0); }

namespace sd {

static std::atomic<uint64_t> g_launches{0};
static std::atomic<uint64_t> g_wait_limit{1000000000ull};
static std::atomic<int32_t> g_index_check{0};

constexpr int kMaxDevices = 64;
static int* g_status_addr[kMaxDevices] = {nullptr};
static std::mutex g_mu;

int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    g_status_addr[dev] = static_cast<int*>(p);
  }
  return g_status_addr[dev];
}

safedit_status after_launch(int n) {
  g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? SAFEDIT_OK : SAFEDIT_ERR_CUDA;
}

uint64_t wait_limit_ns() { return g_wait_limit.load(std::memory_order_relaxed); }

bool index_check_enabled() { return g_index_check.load(std::memory_order_relaxed) != 0; }

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

safedit_status encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                           const uint64_t* dims, const uint64_t* strides_bytes,
                           const uint32_t* box, CUtensorMapSwizzle swizzle) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                           &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return SAFEDIT_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(map, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                        reinterpret_cast<const cuuint64_t*>(dims),
                        reinterpret_cast<const cuuint64_t*>(strides_bytes),
                        reinterpret_cast<const cuuint32_t*>(box), elem_strides,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SAFEDIT_OK : SAFEDIT_ERR_CUDA;
}

safedit_status set_smem(const void* kernel, int bytes) {
  static std::unordered_map<const void*, uint64_t> done;  // kernel -> device bitmask
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAFEDIT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  uint64_t& mask = done[kernel];
  if (mask & (uint64_t(1) << dev)) return SAFEDIT_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return SAFEDIT_ERR_CUDA;
  mask |= uint64_t(1) << dev;
  return SAFEDIT_OK;
}

}  // namespace sd

extern "C" {

safedit_status safedit_get_device_status(int32_t* host_status, void* stream) {
  if (!host_status) return SAFEDIT_ERR_INVALID_ARG;
  if (!sd::status_ptr()) return SAFEDIT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  status_take_kernel<<<1, 1, 0, s>>>();
  if (sd::after_launch(1) != SAFEDIT_OK) return SAFEDIT_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status_taken, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return SAFEDIT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SAFEDIT_ERR_CUDA;
  *host_status = v;
  return SAFEDIT_OK;
}

const char* safedit_status_string(safedit_status st) {
  switch (st) {
    case SAFEDIT_OK: return "ok";
    case SAFEDIT_ERR_INVALID_ARG: return "invalid argument";
    case SAFEDIT_ERR_SHAPE: return "shape mismatch";
    case SAFEDIT_ERR_DTYPE: return "unsupported dtype";
    case SAFEDIT_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case SAFEDIT_ERR_INDEX: return "index out of range";
    case SAFEDIT_ERR_UNSUPPORTED: return "unsupported configuration";
    case SAFEDIT_ERR_CUDA: return "CUDA runtime or driver error";
    case SAFEDIT_ERR_TIMEOUT: return "bounded on-device wait timed out";
    case SAFEDIT_ERR_MASKED_ROW: return "row with no admissible key";
    default: return "unknown status";
  }
}

uint64_t safedit_kernel_launch_count(void) { return sd::g_launches.load(); }

uint64_t safedit_debug_set_wait_limit_ns(uint64_t ns) { return sd::g_wait_limit.exchange(ns); }

int32_t safedit_debug_set_index_check(int32_t on) { return sd::g_index_check.exchange(on ? 1 : 0); }

}  // extern "C"
