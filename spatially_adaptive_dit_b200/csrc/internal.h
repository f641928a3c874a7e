// internal.h -- host-side helpers shared by the translation units of
// libsafedit.so: argument checks, the device status word, the launch counter
// and TMA descriptor encoding.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/safedit.h"

namespace sd {

inline int elt_size(int dtype) {
  switch (dtype) {
    case SAFEDIT_F32: return 4;
    case SAFEDIT_BF16: return 2;
    case SAFEDIT_F16: return 2;
    case SAFEDIT_BOOL: return 1;
    case SAFEDIT_I32: return 4;
    case SAFEDIT_F64: return 8;
    case SAFEDIT_U8: return 1;
    default: return 0;
  }
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Basic structural check of a tensor argument: non-null descriptor, known
// dtype, ndim as expected, non-negative dims, and a data pointer unless the
// tensor is empty (an empty tensor may carry a null pointer; every entry point
// returns before launching anything when its work is empty).
inline safedit_status check_tensor(const safedit_tensor* t, int ndim) {
  if (!t) return SAFEDIT_ERR_INVALID_ARG;
  if (elt_size(t->dtype) == 0) return SAFEDIT_ERR_DTYPE;
  if (t->ndim != ndim || ndim < 1 || ndim > 4) return SAFEDIT_ERR_SHAPE;
  bool empty = false;
  for (int i = 0; i < ndim; ++i) {
    if (t->dims[i] < 0) return SAFEDIT_ERR_SHAPE;
    empty = empty || t->dims[i] == 0;
  }
  if (!t->data && !empty) return SAFEDIT_ERR_INVALID_ARG;
  return SAFEDIT_OK;
}

// Device address of this device's status word (cudaGetSymbolAddress, cached
// per device).  nullptr on failure.
int* status_ptr();

// Launch bookkeeping: adds n to the process-wide kernel launch counter and
// converts the last launch error into a status.
safedit_status after_launch(int n);

uint64_t wait_limit_ns();

// Debug mode (safedit_debug_set_index_check): index vectors that scatter
// rows are checked for duplicates before the scattering kernel runs.
bool index_check_enabled();

// Launches the duplicate / range check of d_idx[0, n_idx) against
// [0, n_rows): one CTA with a bitmap of the row range in shared memory
// (windows of 1.8 M rows), a duplicate or out-of-range entry sets
// SAFEDIT_ERR_INDEX in the status word.  Needs no memory beyond the CTA's.
safedit_status launch_index_check(const int32_t* d_idx, int32_t n_idx, int64_t n_rows, int* status,
                                  cudaStream_t stream);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).  dims/box are innermost first; strides_bytes has rank-1
// entries (dims 1..rank-1).
safedit_status encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                           const uint64_t* dims, const uint64_t* strides_bytes,
                           const uint32_t* box, CUtensorMapSwizzle swizzle);

// Opt a kernel into `bytes` of dynamic shared memory (done once per kernel).
safedit_status set_smem(const void* kernel, int bytes);

}  // namespace sd
