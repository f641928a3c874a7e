// rows_cfg.cu -- the bandwidth kernels of the state update and the guidance
// combine:
//   * scatter_state / gather_rows: indexed row copies of up to four
//     [B,H,rows,d] tensors in one launch (SAFE-DiT summary, 방법론 3: cached
//     context states, refreshed sensitive rows), 16-byte vector accesses,
//     every row a contiguous run so that a warp touches whole lines;
//   * the debug-mode index check: every entry of a scattering index vector
//     in range and no two equal (a duplicate would make two writers race
//     for one row);
//   * sw_cfg: gamma_i = gamma_ctx + (gamma_sens - gamma_ctx) s_i and
//     out = u + gamma_i (c - u) (SAFE-DiT summary, 방법론 4), one fp32 FMA
//     chain per element on 128-bit loads.
#include "common.cuh"
#include "internal.h"

namespace sd {

constexpr int kMaxRowTensors = 4;

struct RowCopyParams {
  const char* src[kMaxRowTensors];
  char* dst[kMaxRowTensors];
  // byte strides of the compact side (b, h, row) and of the indexed side
  int64_t c_sb[kMaxRowTensors], c_sh[kMaxRowTensors], c_sr[kMaxRowTensors];
  int64_t x_sb[kMaxRowTensors], x_sh[kMaxRowTensors], x_sr[kMaxRowTensors];
  int H[kMaxRowTensors], BH[kMaxRowTensors], units[kMaxRowTensors];
  int rows_per_pass[kMaxRowTensors];
  int slices[kMaxRowTensors];  // column slices of kRowThreads units (rows wider than a block)
  int n_idx;       // compact rows
  int n_rows_x;    // rows of the indexed side
  const int* idx;
  int scatter;     // 1: compact -> indexed; 0: indexed -> compact
  int* status;
};

constexpr int kRowThreads = 256;
constexpr int kRowIters = 4;  // independent 16-byte copies in flight per thread

// grid: x = row blocks x column slices, y = b*H + h, z = tensor.  A row of
// at most kRowThreads 16-byte units is one slice, and a block copies several
// such rows per pass; a wider row is cut into slices of kRowThreads units.
// Scattering, a thread's compact-row loads go out before its index loads.
__global__ void __launch_bounds__(kRowThreads) row_copy_kernel(RowCopyParams p) {
  const int t = blockIdx.z;
  const int bh = blockIdx.y;
  if (bh >= p.BH[t]) return;
  const int S = p.slices[t];
  const int xb = blockIdx.x / S, sl = blockIdx.x - xb * S;
  const int Uw = min(p.units[t] - sl * kRowThreads, kRowThreads);
  const int rpp = p.rows_per_pass[t];
  const int sub = threadIdx.x / Uw;
  const int unit = sl * kRowThreads + (threadIdx.x - sub * Uw);
  if (sub >= rpp) return;
  const int b = bh / p.H[t], h = bh - b * p.H[t];
  const char* cb_src;
  char* cb_dst;
  const int64_t c_off = b * p.c_sb[t] + h * p.c_sh[t] + int64_t(unit) * 16;
  const int64_t x_off = b * p.x_sb[t] + h * p.x_sh[t] + int64_t(unit) * 16;
  const int r_base = xb * (rpp * kRowIters) + sub;

  uint4 v[kRowIters];
  int64_t dst_off[kRowIters];
  bool ok[kRowIters];
  if (p.scatter) {
    // the compact rows do not depend on the index: their loads go out first
#pragma unroll
    for (int it = 0; it < kRowIters; ++it) {
      const int r = r_base + it * rpp;
      ok[it] = r < p.n_idx;
      if (ok[it]) v[it] = __ldcs(reinterpret_cast<const uint4*>(p.src[t] + c_off + int64_t(r) * p.c_sr[t]));
    }
#pragma unroll
    for (int it = 0; it < kRowIters; ++it) {
      if (!ok[it]) continue;
      const int r = r_base + it * rpp;
      const int i = __ldg(p.idx + r);
      if (i < 0 || i >= p.n_rows_x) {
        set_status(p.status, SAFEDIT_ERR_INDEX);
        ok[it] = false;
        continue;
      }
      dst_off[it] = x_off + int64_t(i) * p.x_sr[t];
    }
  } else {
#pragma unroll
    for (int it = 0; it < kRowIters; ++it) {
      const int r = r_base + it * rpp;
      ok[it] = r < p.n_idx;
      if (!ok[it]) continue;
      const int i = __ldg(p.idx + r);
      if (i < 0 || i >= p.n_rows_x) {
        set_status(p.status, SAFEDIT_ERR_INDEX);
        ok[it] = false;
        continue;
      }
      cb_src = p.src[t] + x_off + int64_t(i) * p.x_sr[t];
      v[it] = __ldcs(reinterpret_cast<const uint4*>(cb_src));
      dst_off[it] = c_off + int64_t(r) * p.c_sr[t];
    }
  }
#pragma unroll
  for (int it = 0; it < kRowIters; ++it) {
    if (!ok[it]) continue;
    cb_dst = p.dst[t] + dst_off[it];
    *reinterpret_cast<uint4*>(cb_dst) = v[it];
  }
}

// ------------------------------------------------------------ index check
constexpr int kIdxThreads = 1024;
constexpr int kIdxWords = 58112;  // 227 KB of bitmap: 1,859,584 rows per window

// One CTA.  For each window of the row range: clear the bitmap, mark every
// index in the window with an atomic OR (a bit already set is a duplicate),
// repeat.  Out-of-range entries are flagged on the first window.
__global__ void __launch_bounds__(kIdxThreads) index_check_kernel(const int32_t* idx, int32_t n_idx,
                                                                   int64_t n_rows, int words,
                                                                   int* status) {
  extern __shared__ uint32_t bm[];
  const int64_t span = int64_t(words) * 32;
  for (int64_t base = 0; base < n_rows; base += span) {
    for (int w = threadIdx.x; w < words; w += kIdxThreads) bm[w] = 0u;
    __syncthreads();
    bool bad = false;
    for (int r = threadIdx.x; r < n_idx; r += kIdxThreads) {
      const int64_t i = __ldg(idx + r);
      if (i < 0 || i >= n_rows) {
        bad |= (base == 0);
        continue;
      }
      const int64_t off = i - base;
      if (off < 0 || off >= span) continue;
      const uint32_t bit = 1u << (off & 31);
      bad |= (atomicOr(&bm[off >> 5], bit) & bit) != 0u;
    }
    if (bad) set_status(status, SAFEDIT_ERR_INDEX);
    __syncthreads();
  }
}

safedit_status launch_index_check(const int32_t* d_idx, int32_t n_idx, int64_t n_rows, int* status,
                                  cudaStream_t stream) {
  if (n_idx <= 0 || n_rows <= 0) return SAFEDIT_OK;
  const int64_t need = (n_rows + 31) / 32;
  const int words = static_cast<int>(need < kIdxWords ? need : kIdxWords);
  const int bytes = words * 4;
  static_assert(kIdxWords * 4 <= 232448, "bitmap");
  safedit_status st = set_smem(reinterpret_cast<const void*>(index_check_kernel), kIdxWords * 4);
  if (st != SAFEDIT_OK) return st;
  index_check_kernel<<<1, kIdxThreads, bytes, stream>>>(d_idx, n_idx, n_rows, words, status);
  return after_launch(1);
}

static safedit_status row_copy(const safedit_tensor* src, const safedit_tensor* dst, int n_tensors,
                               const int32_t* d_idx, int32_t n_idx, void* stream, int scatter) {
  if (!src || !dst || n_tensors < 1 || n_tensors > kMaxRowTensors || n_idx < 0)
    return SAFEDIT_ERR_INVALID_ARG;
  if (n_idx > 0 && !d_idx) return SAFEDIT_ERR_INVALID_ARG;
  RowCopyParams p{};
  int max_bh = 0, max_blocks = 0;
  int n_rows_x = -1;
  for (int t = 0; t < n_tensors; ++t) {
    const safedit_tensor& s = src[t];
    const safedit_tensor& d = dst[t];
    safedit_status st;
    if ((st = check_tensor(&s, 4)) != SAFEDIT_OK) return st;
    if ((st = check_tensor(&d, 4)) != SAFEDIT_OK) return st;
    if (s.dtype != d.dtype) return SAFEDIT_ERR_DTYPE;
    const int es = elt_size(s.dtype);
    if (es != 2 && es != 4) return SAFEDIT_ERR_DTYPE;
    const safedit_tensor& compact = scatter ? s : d;
    const safedit_tensor& indexed = scatter ? d : s;
    if (compact.dims[0] != indexed.dims[0] || compact.dims[1] != indexed.dims[1] ||
        compact.dims[3] != indexed.dims[3])
      return SAFEDIT_ERR_SHAPE;
    if (compact.dims[2] != n_idx) return SAFEDIT_ERR_SHAPE;
    if (n_rows_x < 0) n_rows_x = static_cast<int>(indexed.dims[2]);
    if (indexed.dims[2] != n_rows_x) return SAFEDIT_ERR_SHAPE;
    if (s.strides[3] != 1 || d.strides[3] != 1) return SAFEDIT_ERR_ALIGNMENT;
    const int64_t row_bytes = s.dims[3] * es;
    if (row_bytes % 16 != 0 || row_bytes == 0) return SAFEDIT_ERR_ALIGNMENT;
    for (int k = 0; k < 3; ++k)
      if ((s.strides[k] * es) % 16 != 0 || (d.strides[k] * es) % 16 != 0)
        return SAFEDIT_ERR_ALIGNMENT;
    if (!aligned16(s.data) || !aligned16(d.data)) return SAFEDIT_ERR_ALIGNMENT;
    if (s.dims[0] * s.dims[1] > 65535) return SAFEDIT_ERR_UNSUPPORTED;
    p.src[t] = static_cast<const char*>(s.data);
    p.dst[t] = static_cast<char*>(d.data);
    p.c_sb[t] = compact.strides[0] * es;
    p.c_sh[t] = compact.strides[1] * es;
    p.c_sr[t] = compact.strides[2] * es;
    p.x_sb[t] = indexed.strides[0] * es;
    p.x_sh[t] = indexed.strides[1] * es;
    p.x_sr[t] = indexed.strides[2] * es;
    p.H[t] = static_cast<int>(s.dims[1]);
    p.BH[t] = static_cast<int>(s.dims[0] * s.dims[1]);
    p.units[t] = static_cast<int>(row_bytes / 16);
    if (row_bytes / 16 > INT32_MAX / 2) return SAFEDIT_ERR_UNSUPPORTED;
    p.slices[t] = (p.units[t] + kRowThreads - 1) / kRowThreads;
    p.rows_per_pass[t] = p.slices[t] > 1 ? 1 : kRowThreads / p.units[t];
    const int rows_per_block = p.rows_per_pass[t] * kRowIters;
    const int64_t blocks64 = int64_t((n_idx + rows_per_block - 1) / rows_per_block) * p.slices[t];
    if (blocks64 > INT32_MAX) return SAFEDIT_ERR_UNSUPPORTED;
    const int blocks = static_cast<int>(blocks64);
    if (p.BH[t] > max_bh) max_bh = p.BH[t];
    if (blocks > max_blocks) max_blocks = blocks;
  }
  if (n_idx == 0 || max_bh == 0) return SAFEDIT_OK;
  p.n_idx = n_idx;
  p.n_rows_x = n_rows_x;
  p.idx = d_idx;
  p.scatter = scatter;
  p.status = status_ptr();
  if (!p.status) return SAFEDIT_ERR_CUDA;
  if (scatter && index_check_enabled()) {
    const safedit_status st = launch_index_check(d_idx, n_idx, n_rows_x, p.status,
                                                 static_cast<cudaStream_t>(stream));
    if (st != SAFEDIT_OK) return st;
  }
  dim3 grid(max_blocks, max_bh, n_tensors);
  row_copy_kernel<<<grid, kRowThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return after_launch(1);
}

// --------------------------------------------------------------- sw_cfg ---
struct CfgParams {
  const void* c;    // f32 or bf16 (the template parameter of the kernel)
  const void* u;
  const float* s;
  float* out;
  int64_t N, F;
  int64_t sc, su, so;  // row strides (elements)
  float g_ctx, g_diff;
};

// Four consecutive predictions as floats (bf16 widened exactly), streamed.
__device__ __forceinline__ float4 load4_cs(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ float4 load4_cs(const __nv_bfloat16* p) {
  const uint2 v = __ldcs(reinterpret_cast<const uint2*>(p));
  return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                     __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
}
__device__ __forceinline__ float load1(const float* p) { return *p; }
__device__ __forceinline__ float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__global__ void __launch_bounds__(256) sw_cfg_vec4_kernel(CfgParams p) {
  const T* pc = static_cast<const T*>(p.c);
  const T* pu = static_cast<const T*>(p.u);
  const int64_t F4 = p.F >> 2;
  const int64_t total = p.N * F4;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t i = e / F4;
    const int64_t f = (e - i * F4) << 2;
    const float g = fmaf(p.g_diff, __ldg(p.s + i), p.g_ctx);
    const float4 c = load4_cs(pc + i * p.sc + f);
    const float4 u = load4_cs(pu + i * p.su + f);
    float4 o;
    o.x = fmaf(g, c.x - u.x, u.x);
    o.y = fmaf(g, c.y - u.y, u.y);
    o.z = fmaf(g, c.z - u.z, u.z);
    o.w = fmaf(g, c.w - u.w, u.w);
    __stcs(reinterpret_cast<float4*>(p.out + i * p.so + f), o);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) sw_cfg_scalar_kernel(CfgParams p) {
  const T* pc = static_cast<const T*>(p.c);
  const T* pu = static_cast<const T*>(p.u);
  const int64_t total = p.N * p.F;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t i = e / p.F;
    const int64_t f = e - i * p.F;
    const float g = fmaf(p.g_diff, p.s[i], p.g_ctx);
    const float c = load1(pc + i * p.sc + f), u = load1(pu + i * p.su + f);
    p.out[i * p.so + f] = fmaf(g, c - u, u);
  }
}

// ------------------------------------------------------------ StepCache ---
// AccelAes summary B.3: between full steps the noise prediction is reused by
// linear extrapolation; fused with the guidance combine:
//   c = c_b + w (c_b - c_a),  u = u_b + w (u_b - u_a),  out = u + gamma_i (c - u).
struct StepCacheParams {
  const float* ca;
  const float* cb;
  const float* ua;
  const float* ub;
  const float* s;
  float* out;
  int64_t N, F;
  int64_t sca, scb, sua, sub, so;  // row strides (elements)
  float w, g_ctx, g_diff;
};

__device__ __forceinline__ float stepcache_one(float ca, float cb, float ua, float ub, float w,
                                               float g) {
  const float c = fmaf(w, cb - ca, cb);
  const float u = fmaf(w, ub - ua, ub);
  return fmaf(g, c - u, u);
}

__global__ void __launch_bounds__(256) stepcache_vec4_kernel(StepCacheParams p) {
  const int64_t F4 = p.F >> 2;
  const int64_t total = p.N * F4;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t i = e / F4;
    const int64_t f = (e - i * F4) << 2;
    const float g = fmaf(p.g_diff, __ldg(p.s + i), p.g_ctx);
    const float4 ca = __ldcs(reinterpret_cast<const float4*>(p.ca + i * p.sca + f));
    const float4 cb = __ldcs(reinterpret_cast<const float4*>(p.cb + i * p.scb + f));
    const float4 ua = __ldcs(reinterpret_cast<const float4*>(p.ua + i * p.sua + f));
    const float4 ub = __ldcs(reinterpret_cast<const float4*>(p.ub + i * p.sub + f));
    float4 o;
    o.x = stepcache_one(ca.x, cb.x, ua.x, ub.x, p.w, g);
    o.y = stepcache_one(ca.y, cb.y, ua.y, ub.y, p.w, g);
    o.z = stepcache_one(ca.z, cb.z, ua.z, ub.z, p.w, g);
    o.w = stepcache_one(ca.w, cb.w, ua.w, ub.w, p.w, g);
    __stcs(reinterpret_cast<float4*>(p.out + i * p.so + f), o);
  }
}

__global__ void __launch_bounds__(256) stepcache_scalar_kernel(StepCacheParams p) {
  const int64_t total = p.N * p.F;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t i = e / p.F;
    const int64_t f = e - i * p.F;
    const float g = fmaf(p.g_diff, p.s[i], p.g_ctx);
    p.out[i * p.so + f] = stepcache_one(p.ca[i * p.sca + f], p.cb[i * p.scb + f],
                                        p.ua[i * p.sua + f], p.ub[i * p.sub + f], p.w, g);
  }
}

}  // namespace sd

using namespace sd;

extern "C" {

safedit_status safedit_scatter_state(const safedit_tensor* src, const safedit_tensor* dst,
                                     int32_t n_tensors, const int32_t* d_idx, int32_t n_idx,
                                     void* stream) {
  return row_copy(src, dst, n_tensors, d_idx, n_idx, stream, 1);
}

safedit_status safedit_gather_rows(const safedit_tensor* src, const safedit_tensor* dst,
                                   int32_t n_tensors, const int32_t* d_idx, int32_t n_idx,
                                   void* stream) {
  return row_copy(src, dst, n_tensors, d_idx, n_idx, stream, 0);
}

safedit_status safedit_sw_cfg(const safedit_tensor* eps_c, const safedit_tensor* eps_u,
                              const float* d_s, float gamma_ctx, float gamma_sens,
                              const safedit_tensor* out, void* stream) {
  safedit_status st;
  if ((st = check_tensor(eps_c, 2)) != SAFEDIT_OK) return st;
  if ((st = check_tensor(eps_u, 2)) != SAFEDIT_OK) return st;
  if ((st = check_tensor(out, 2)) != SAFEDIT_OK) return st;
  const bool bf16 = eps_c->dtype == SAFEDIT_BF16;
  if ((eps_c->dtype != SAFEDIT_F32 && !bf16) || eps_u->dtype != eps_c->dtype || out->dtype != SAFEDIT_F32)
    return SAFEDIT_ERR_DTYPE;
  const int64_t N = eps_c->dims[0], F = eps_c->dims[1];
  if (eps_u->dims[0] != N || eps_u->dims[1] != F || out->dims[0] != N || out->dims[1] != F)
    return SAFEDIT_ERR_SHAPE;
  if (eps_c->strides[1] != 1 || eps_u->strides[1] != 1 || out->strides[1] != 1)
    return SAFEDIT_ERR_ALIGNMENT;
  if (N == 0 || F == 0) return SAFEDIT_OK;
  if (!d_s) return SAFEDIT_ERR_INVALID_ARG;
  CfgParams p;
  p.c = eps_c->data;
  p.u = eps_u->data;
  p.s = d_s;
  p.out = static_cast<float*>(out->data);
  p.N = N;
  p.F = F;
  p.sc = eps_c->strides[0];
  p.su = eps_u->strides[0];
  p.so = out->strides[0];
  p.g_ctx = gamma_ctx;
  p.g_diff = gamma_sens - gamma_ctx;
  // 4 predictions per thread: 16-byte (f32) or 8-byte (bf16) aligned groups
  const uintptr_t in_align = bf16 ? 7u : 15u;
  const bool vec = (F % 4 == 0) && (p.sc % 4 == 0) && (p.su % 4 == 0) && (p.so % 4 == 0) &&
                   (reinterpret_cast<uintptr_t>(p.c) & in_align) == 0 &&
                   (reinterpret_cast<uintptr_t>(p.u) & in_align) == 0 && aligned16(p.out);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t work = vec ? N * (F / 4) : N * F;
  int64_t blocks = (work + 255) / 256;
  const int64_t cap = int64_t(sms) * 8;
  if (blocks > cap) blocks = cap;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>(blocks);
  if (vec && bf16)
    sw_cfg_vec4_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
  else if (vec)
    sw_cfg_vec4_kernel<float><<<grid, 256, 0, s>>>(p);
  else if (bf16)
    sw_cfg_scalar_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
  else
    sw_cfg_scalar_kernel<float><<<grid, 256, 0, s>>>(p);
  return after_launch(1);
}

safedit_status safedit_stepcache_sw_cfg(const safedit_tensor* eps_c_a, const safedit_tensor* eps_c_b,
                                        const safedit_tensor* eps_u_a, const safedit_tensor* eps_u_b,
                                        const float* d_s, float w, float gamma_ctx, float gamma_sens,
                                        const safedit_tensor* out, void* stream) {
  safedit_status st;
  const safedit_tensor* ins[4] = {eps_c_a, eps_c_b, eps_u_a, eps_u_b};
  for (const safedit_tensor* t : ins)
    if ((st = check_tensor(t, 2)) != SAFEDIT_OK) return st;
  if ((st = check_tensor(out, 2)) != SAFEDIT_OK) return st;
  const int64_t N = out->dims[0], F = out->dims[1];
  for (const safedit_tensor* t : ins) {
    if (t->dtype != SAFEDIT_F32) return SAFEDIT_ERR_DTYPE;
    if (t->dims[0] != N || t->dims[1] != F) return SAFEDIT_ERR_SHAPE;
    if (t->strides[1] != 1) return SAFEDIT_ERR_ALIGNMENT;
  }
  if (out->dtype != SAFEDIT_F32) return SAFEDIT_ERR_DTYPE;
  if (out->strides[1] != 1) return SAFEDIT_ERR_ALIGNMENT;
  if (N == 0 || F == 0) return SAFEDIT_OK;
  if (!d_s) return SAFEDIT_ERR_INVALID_ARG;
  StepCacheParams p;
  p.ca = static_cast<const float*>(eps_c_a->data);
  p.cb = static_cast<const float*>(eps_c_b->data);
  p.ua = static_cast<const float*>(eps_u_a->data);
  p.ub = static_cast<const float*>(eps_u_b->data);
  p.s = d_s;
  p.out = static_cast<float*>(out->data);
  p.N = N;
  p.F = F;
  p.sca = eps_c_a->strides[0];
  p.scb = eps_c_b->strides[0];
  p.sua = eps_u_a->strides[0];
  p.sub = eps_u_b->strides[0];
  p.so = out->strides[0];
  p.w = w;
  p.g_ctx = gamma_ctx;
  p.g_diff = gamma_sens - gamma_ctx;
  bool vec = (F % 4 == 0) && aligned16(p.out) && (p.so % 4 == 0);
  for (const safedit_tensor* t : ins) vec = vec && aligned16(t->data) && (t->strides[0] % 4 == 0);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t work = vec ? N * (F / 4) : N * F;
  int64_t blocks = (work + 255) / 256;
  const int64_t cap = int64_t(sms) * 8;
  if (blocks > cap) blocks = cap;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (vec)
    stepcache_vec4_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(p);
  else
    stepcache_scalar_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(p);
  return after_launch(1);
}

}  // extern "C"
