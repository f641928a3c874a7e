// mask.cu -- the exact mask-elision criterion (SAFE-DiT summary, 방법론 1;
// Italian page, Metodologia 1): an additive mask row may be dropped iff it
// is a constant shift c_i of the logits, i.e. all entries equal entry 0 under
// IEEE == and that entry is finite.  One warp per row, 128-bit loads, an
// integer fast path (bit-identical words) with an IEEE fallback (+0 vs -0),
// a warp vote per row, and an early exit once any row is kept (when per-row
// flags are not requested).
#include "common.cuh"
#include "internal.h"

namespace sd {

struct MaskParams {
  const char* base;
  int dtype;
  int64_t B, Hm, Nq, Nk;
  int64_t sb, sh, sq, sk;  // element strides
  int* verdict;
  uint8_t* row_flags;      // nullable, [B*Hm*Nq]
  int vec;                 // 16-byte vector path usable
};

constexpr int kMaskWarps = 8;

__global__ void mask_init_kernel(int* verdict) { *verdict = 1; }

__device__ __forceinline__ bool finite_bits(uint32_t v, int dtype) {
  switch (dtype) {
    case SAFEDIT_F32: return (v & 0x7F800000u) != 0x7F800000u;
    case SAFEDIT_BF16: return (v & 0x7F80u) != 0x7F80u;
    case SAFEDIT_F16: return (v & 0x7C00u) != 0x7C00u;
    default: return v != 0u;  // bool: true (attend) is the finite value 0
  }
}

// IEEE equality of one element (given as raw bits) with the row's first
// element v0, which is known to be finite.
__device__ __forceinline__ bool elt_equal(uint32_t x, uint32_t v0, int dtype) {
  switch (dtype) {
    case SAFEDIT_F32: return __uint_as_float(x) == __uint_as_float(v0);
    case SAFEDIT_BF16: return x == v0 || ((x | v0) & 0x7FFFu) == 0u;
    case SAFEDIT_F16: return x == v0 || ((x | v0) & 0x7FFFu) == 0u;
    default: return x != 0u;  // bool: every entry must be true
  }
}

__device__ __forceinline__ uint32_t load_elt(const char* p, int dtype) {
  switch (dtype) {
    case SAFEDIT_F32: return *reinterpret_cast<const uint32_t*>(p);
    case SAFEDIT_BF16:
    case SAFEDIT_F16: return *reinterpret_cast<const uint16_t*>(p);
    default: return *reinterpret_cast<const uint8_t*>(p);
  }
}

// Checks one 16-byte word group against v0; returns true if all equal.
__device__ __forceinline__ bool vec_equal(uint4 w, uint32_t v0, int dtype) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  bool ok = true;
  if (dtype == SAFEDIT_F32) {
#pragma unroll
    for (int k = 0; k < 4; ++k) ok &= elt_equal(ws[k], v0, dtype);
  } else if (dtype == SAFEDIT_BOOL) {
#pragma unroll
    for (int k = 0; k < 4; ++k) ok &= ((ws[k] - 0x01010101u) & ~ws[k] & 0x80808080u) == 0u;
  } else {
    const uint32_t pair = v0 | (v0 << 16);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (ws[k] != pair) {
        ok &= elt_equal(ws[k] & 0xFFFFu, v0, dtype);
        ok &= elt_equal(ws[k] >> 16, v0, dtype);
      }
    }
  }
  return ok;
}

__global__ void __launch_bounds__(kMaskWarps * 32) mask_rows_kernel(MaskParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t nrows = p.B * p.Hm * p.Nq;
  const int64_t nwarps = int64_t(gridDim.x) * kMaskWarps;
  const int es = p.dtype == SAFEDIT_F32 ? 4 : (p.dtype == SAFEDIT_BOOL ? 1 : 2);
  for (int64_t row = blockIdx.x * int64_t(kMaskWarps) + (threadIdx.x >> 5); row < nrows;
       row += nwarps) {
    // warp-uniform exit once another row has been found kept
    if (!p.row_flags &&
        __any_sync(0xffffffffu, *reinterpret_cast<volatile int*>(p.verdict) == 0))
      return;
    const int64_t q = row % p.Nq;
    const int64_t bh = row / p.Nq;
    const int64_t h = bh % p.Hm, b = bh / p.Hm;
    const char* rp = p.base + (b * p.sb + h * p.sh + q * p.sq) * es;
    const uint32_t v0 = load_elt(rp, p.dtype);
    bool ok = finite_bits(v0, p.dtype);
    if (ok) {
      if (p.vec) {
        const int64_t nv = (p.Nk * es) >> 4;  // 16-byte words in the row
        const uint4* w = reinterpret_cast<const uint4*>(rp);
        int64_t j = lane;
        for (; j + 96 < nv; j += 128) {
          const uint4 a = __ldcs(w + j), b2 = __ldcs(w + j + 32), c = __ldcs(w + j + 64),
                      d = __ldcs(w + j + 96);
          ok &= vec_equal(a, v0, p.dtype) & vec_equal(b2, v0, p.dtype) &
                vec_equal(c, v0, p.dtype) & vec_equal(d, v0, p.dtype);
        }
        for (; j < nv; j += 32) ok &= vec_equal(__ldcs(w + j), v0, p.dtype);
      } else {
        for (int64_t j = lane; j < p.Nk; j += 32)
          ok &= elt_equal(load_elt(rp + j * p.sk * es, p.dtype), v0, p.dtype);
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    if (lane == 0) {
      if (p.row_flags) p.row_flags[row] = ok ? 1 : 0;
      // one store clears the verdict: thousands of warps storing to the same
      // word would serialise in L2
      if (!ok && *reinterpret_cast<volatile int*>(p.verdict) != 0) *p.verdict = 0;
    }
  }
}

}  // namespace sd

using namespace sd;

extern "C" safedit_status safedit_mask_is_row_constant(const safedit_tensor* mask,
                                                       int32_t* d_verdict, uint8_t* d_row_flags,
                                                       void* stream) {
  if (!mask || !mask->data || !d_verdict) return SAFEDIT_ERR_INVALID_ARG;
  if (mask->ndim < 2 || mask->ndim > 4) return SAFEDIT_ERR_SHAPE;
  const int dt = mask->dtype;
  if (dt != SAFEDIT_F32 && dt != SAFEDIT_BF16 && dt != SAFEDIT_F16 && dt != SAFEDIT_BOOL)
    return SAFEDIT_ERR_DTYPE;
  int64_t dims[4] = {1, 1, 1, 1}, strides[4] = {0, 0, 0, 0};
  const int off = 4 - mask->ndim;
  for (int i = 0; i < mask->ndim; ++i) {
    if (mask->dims[i] < 0) return SAFEDIT_ERR_SHAPE;
    dims[off + i] = mask->dims[i];
    strides[off + i] = mask->strides[i];
  }
  if (dims[3] == 0) return SAFEDIT_ERR_SHAPE;
  if (strides[3] != 0 && strides[3] != 1) return SAFEDIT_ERR_ALIGNMENT;
  MaskParams p;
  p.base = static_cast<const char*>(mask->data);
  p.dtype = dt;
  p.B = dims[0];
  p.Hm = dims[1];
  p.Nq = dims[2];
  p.Nk = dims[3];
  p.sb = strides[0];
  p.sh = strides[1];
  p.sq = strides[2];
  p.sk = strides[3];
  p.verdict = d_verdict;
  p.row_flags = d_row_flags;
  // Without per-row flags, rows that are the same memory (broadcast dims)
  // are checked once.
  if (!d_row_flags) {
    if (p.sb == 0) p.B = 1;
    if (p.sh == 0) p.Hm = 1;
    if (p.sq == 0) p.Nq = 1;
  }
  const int es = elt_size(dt);
  p.vec = (p.sk == 1) && ((p.Nk * es) % 16 == 0) && aligned16(p.base) &&
          ((p.sb * es) % 16 == 0) && ((p.sh * es) % 16 == 0) && ((p.sq * es) % 16 == 0);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  mask_init_kernel<<<1, 1, 0, s>>>(d_verdict);
  const int64_t nrows = p.B * p.Hm * p.Nq;
  if (nrows == 0) return after_launch(1);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (nrows + kMaskWarps - 1) / kMaskWarps;
  const int64_t cap = int64_t(sms) * 8;
  if (blocks > cap) blocks = cap;
  mask_rows_kernel<<<static_cast<unsigned>(blocks), kMaskWarps * 32, 0, s>>>(p);
  return after_launch(2);
}
