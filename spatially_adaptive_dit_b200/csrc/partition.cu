// partition.cu -- PCSP (SAFE-DiT summary, 방법론 2; AccelAes summary B.1):
//   * partition_accumulate: score[i] += sum_h sum_{content j} P[h,i,j] (P in
//     f32 or bf16), one warp per image token, 128-bit streaming loads of the
//     16-byte groups of P that hold a content column (padding is never
//     read), fp64 accumulation and a warp-shuffle reduction;
//   * partition_finalize: the top-k split (ties to the lower index) by an
//     8-pass radix select on order-preserving 64-bit keys, a stable
//     block-scan compaction into ascending S / C index lists, and the
//     min-max sensitivity score s -- one CTA, once per trajectory.
#include "common.cuh"
#include "internal.h"

namespace sd {

// ---------------------------------------------------------- accumulate ----
struct AccParams {
  const void* P;  // f32 or bf16 elements
  const uint8_t* content;
  double* score;
  int64_t H, N, L;
  int64_t sH, sN;  // element strides of P
  int* status;
};

constexpr int kAccWarps = 8;
constexpr int kAccHeads = 4;  // heads whose loads a lane keeps in flight at once (8 measured slower)

// element e of a 16-byte group of P as f32 (bf16 widens exactly)
template <typename T>
__device__ __forceinline__ float acc_elem(const uint4& v, int e);
template <>
__device__ __forceinline__ float acc_elem<float>(const uint4& v, int e) {
  const uint32_t w = e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
  return __uint_as_float(w);
}
template <>
__device__ __forceinline__ float acc_elem<__nv_bfloat16>(const uint4& v, int e) {
  const int q = e >> 1;
  const uint32_t w = q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
  return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

// Vector path: 16-byte groups of VEC = 16 / sizeof(T) columns, L % VEC == 0,
// strides % VEC == 0, 16-byte aligned base, L <= 32 VEC NCH (NCH passes of
// 32 groups per warp).
template <typename T, int NCH>
__global__ void __launch_bounds__(kAccWarps * 32) accumulate_vec_kernel(AccParams p) {
  constexpr int VEC = 16 / int(sizeof(T));
  constexpr int CH = 32 * VEC;  // columns per pass of the warp
  static_assert(VEC * NCH <= 32, "content flags of a lane fit one word");
  const T* const P = static_cast<const T*>(p.P);
  const int lane = threadIdx.x & 31;
  const int64_t warp = blockIdx.x * int64_t(kAccWarps) + (threadIdx.x >> 5);
  const int64_t nwarps = int64_t(gridDim.x) * kAccWarps;
  constexpr uint32_t kGroup = (1u << VEC) - 1u;
  // content flags of this lane's columns: VEC bits per pass
  uint32_t cmask = 0;
  for (int c = 0; c < NCH; ++c)
    for (int e = 0; e < VEC; ++e) {
      const int64_t j = int64_t(c) * CH + lane * VEC + e;
      if (j < p.L && p.content[j]) cmask |= 1u << (c * VEC + e);
    }
  for (int64_t i = warp; i < p.N; i += nwarps) {
    double acc = 0.0;
    const T* row0 = P + i * p.sN;
    int64_t h = 0;
    for (; h + kAccHeads <= p.H; h += kAccHeads) {
      uint4 v[kAccHeads][NCH];
#pragma unroll
      for (int hh = 0; hh < kAccHeads; ++hh)
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          // only 16-byte groups holding a content column are read (text
          // padding and the non-content tokens never leave HBM)
          if ((cmask >> (c * VEC)) & kGroup)
            v[hh][c] = __ldcs(reinterpret_cast<const uint4*>(row0 + (h + hh) * p.sH + int64_t(c) * CH +
                                                             lane * VEC));
          else
            v[hh][c] = make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
      for (int hh = 0; hh < kAccHeads; ++hh)
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          const uint32_t m = cmask >> (c * VEC);
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            if ((m >> e) & 1u) acc += static_cast<double>(acc_elem<T>(v[hh][c], e));
        }
    }
    for (; h < p.H; ++h) {
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const uint32_t m = cmask >> (c * VEC);
        if (m & kGroup) {
          const uint4 v = __ldcs(reinterpret_cast<const uint4*>(row0 + h * p.sH + int64_t(c) * CH + lane * VEC));
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            if ((m >> e) & 1u) acc += static_cast<double>(acc_elem<T>(v, e));
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) p.score[i] += acc;
  }
}

// General path: any L and strides (inner stride 1).
template <typename T>
__global__ void __launch_bounds__(kAccWarps * 32) accumulate_scalar_kernel(AccParams p) {
  const T* const P = static_cast<const T*>(p.P);
  const int lane = threadIdx.x & 31;
  const int64_t warp = blockIdx.x * int64_t(kAccWarps) + (threadIdx.x >> 5);
  const int64_t nwarps = int64_t(gridDim.x) * kAccWarps;
  for (int64_t i = warp; i < p.N; i += nwarps) {
    double acc = 0.0;
    for (int64_t h = 0; h < p.H; ++h) {
      const T* row = P + h * p.sH + i * p.sN;
      for (int64_t j = lane; j < p.L; j += 32)
        if (p.content[j]) acc += static_cast<double>(static_cast<float>(row[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) p.score[i] += acc;
  }
}

// ------------------------------------------------------------ finalize ----
constexpr int kFinThreads = 1024;

// Order-preserving map double -> uint64 (larger score -> larger key); -0 is
// folded onto +0 so that the two compare equal, as they do as doubles.
__device__ __forceinline__ uint64_t score_key(double x) {
  if (x == 0.0) x = 0.0;
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Exclusive block scan of one int per thread (kFinThreads threads); returns
// the exclusive prefix and writes the block total to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int w = warp_sums[lane];
    int s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s - w;  // exclusive prefix of warp totals
    if (lane == 31) *total = s;
  }
  __syncthreads();
  const int r = warp_sums[wid] + x - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kFinThreads, 1)
    finalize_kernel(const double* __restrict__ score, int n, int k, int* __restrict__ idx_s,
                    int* __restrict__ idx_c, float* __restrict__ s_out, int* status) {
  __shared__ unsigned int hist[256];
  __shared__ int warp_sums[32];
  __shared__ int total;
  __shared__ uint64_t sh_prefix;
  __shared__ int sh_need;
  __shared__ double red_lo[32], red_hi[32];
  __shared__ int sh_nan;
  const int tid = threadIdx.x;
  if (tid == 0) sh_nan = 0;
  __syncthreads();

  // min / max (exact, order independent) and the NaN check
  double lo = INFINITY, hi = -INFINITY;
  for (int i = tid; i < n; i += kFinThreads) {
    const double x = score[i];
    if (isnan(x)) sh_nan = 1;
    lo = fmin(lo, x);
    hi = fmax(hi, x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if ((tid & 31) == 0) {
    red_lo[tid >> 5] = lo;
    red_hi[tid >> 5] = hi;
  }
  __syncthreads();
  if (tid < 32) {
    lo = red_lo[tid];
    hi = red_hi[tid];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (tid == 0) {
      red_lo[0] = lo;
      red_hi[0] = hi;
    }
  }
  __syncthreads();
  lo = red_lo[0];
  hi = red_hi[0];
  if (sh_nan && tid == 0) set_status(status, SAFEDIT_ERR_INVALID_ARG);

  // radix select of the k-th largest key (k >= 1), most significant byte first
  uint64_t prefix = 0, pmask = 0;
  int remaining = k;
  if (k > 0 && k < n) {
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int b = tid; b < 256; b += kFinThreads) hist[b] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kFinThreads) {
        const uint64_t key = score_key(score[i]);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFF], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        int cum = 0, sel = 0;
        for (int b = 255; b >= 0; --b) {
          const int c = static_cast<int>(hist[b]);
          if (cum + c >= remaining) {
            sel = b;
            break;
          }
          cum += c;
        }
        sh_prefix = prefix | (uint64_t(sel) << shift);
        sh_need = remaining - cum;
      }
      __syncthreads();
      prefix = sh_prefix;
      remaining = sh_need;
      pmask |= uint64_t(0xFF) << shift;
      __syncthreads();
    }
  }
  // prefix = T, the k-th largest key; `remaining` keys equal to T are taken,
  // those of lowest index.
  const uint64_t T = prefix;
  const int need_eq = remaining;

  int eq_before = 0, sel_before = 0;
  for (int base = 0; base < n; base += kFinThreads) {
    const int i = base + tid;
    const bool in = i < n;
    uint64_t key = 0;
    double x = 0.0;
    if (in) {
      x = score[i];
      key = score_key(x);
    }
    bool sel;
    if (k == 0)
      sel = false;
    else if (k >= n)
      sel = in;
    else {
      const int eq = (in && key == T) ? 1 : 0;
      const int eq_rank = eq_before + block_exclusive_scan(eq, warp_sums, &total);
      eq_before += total;
      sel = in && (key > T || (eq && eq_rank < need_eq));
    }
    const int pos_s = sel_before + block_exclusive_scan(sel ? 1 : 0, warp_sums, &total);
    sel_before += total;
    if (in) {
      if (sel) {
        if (idx_s && pos_s < k) idx_s[pos_s] = i;
      } else {
        if (idx_c && i - pos_s < n - k) idx_c[i - pos_s] = i;
      }
      if (s_out) s_out[i] = (hi == lo) ? 0.0f : __double2float_rn((x - lo) / (hi - lo));
    }
  }
}

}  // namespace sd

using namespace sd;

extern "C" {

safedit_status safedit_partition_accumulate(const safedit_tensor* p, const uint8_t* d_content,
                                            double* d_score, void* stream) {
  safedit_status st;
  if ((st = check_tensor(p, 3)) != SAFEDIT_OK) return st;
  if ((p->dims[2] > 0 && !d_content) || (p->dims[1] > 0 && !d_score))
    return SAFEDIT_ERR_INVALID_ARG;
  if (p->dtype != SAFEDIT_F32 && p->dtype != SAFEDIT_BF16) return SAFEDIT_ERR_DTYPE;
  if (p->strides[2] != 1) return SAFEDIT_ERR_ALIGNMENT;
  const bool bf16 = p->dtype == SAFEDIT_BF16;
  AccParams a;
  a.P = p->data;
  a.content = d_content;
  a.score = d_score;
  a.H = p->dims[0];
  a.N = p->dims[1];
  a.L = p->dims[2];
  a.sH = p->strides[0];
  a.sN = p->strides[1];
  if (a.N == 0) return SAFEDIT_OK;
  a.status = status_ptr();
  if (!a.status) return SAFEDIT_ERR_CUDA;
  const int vec_w = bf16 ? 8 : 4;  // elements per 16-byte group
  const bool vec = (a.L % vec_w == 0) && (a.sH % vec_w == 0) && (a.sN % vec_w == 0) && aligned16(a.P) &&
                   a.L <= 1024;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (a.N + kAccWarps - 1) / kAccWarps;
  const int64_t cap = int64_t(sms) * 16;
  if (blocks > cap) blocks = cap;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nch = static_cast<int>((a.L + 32 * vec_w - 1) / (32 * vec_w));  // passes of 32 groups
  const dim3 grid(static_cast<unsigned>(blocks)), block(kAccWarps * 32);
  if (!vec) {
    if (bf16)
      accumulate_scalar_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(a);
    else
      accumulate_scalar_kernel<float><<<grid, block, 0, s>>>(a);
  } else if (bf16) {
    if (nch <= 1)
      accumulate_vec_kernel<__nv_bfloat16, 1><<<grid, block, 0, s>>>(a);
    else if (nch <= 2)
      accumulate_vec_kernel<__nv_bfloat16, 2><<<grid, block, 0, s>>>(a);
    else
      accumulate_vec_kernel<__nv_bfloat16, 4><<<grid, block, 0, s>>>(a);
  } else {
    if (nch <= 1)
      accumulate_vec_kernel<float, 1><<<grid, block, 0, s>>>(a);
    else if (nch <= 2)
      accumulate_vec_kernel<float, 2><<<grid, block, 0, s>>>(a);
    else if (nch <= 4)
      accumulate_vec_kernel<float, 4><<<grid, block, 0, s>>>(a);
    else
      accumulate_vec_kernel<float, 8><<<grid, block, 0, s>>>(a);
  }
  return after_launch(1);
}

safedit_status safedit_partition_finalize(const double* d_score, int32_t n, int32_t k,
                                          int32_t* d_idx_s, int32_t* d_idx_c, float* d_s,
                                          void* stream) {
  if (n < 0 || k < 0 || k > n || n > (1 << 24)) return SAFEDIT_ERR_INVALID_ARG;
  if (n == 0) return SAFEDIT_OK;
  if (!d_score) return SAFEDIT_ERR_INVALID_ARG;
  int* status = status_ptr();
  if (!status) return SAFEDIT_ERR_CUDA;
  finalize_kernel<<<1, kFinThreads, 0, static_cast<cudaStream_t>(stream)>>>(d_score, n, k, d_idx_s,
                                                                            d_idx_c, d_s, status);
  return after_launch(1);
}

}  // extern "C"
