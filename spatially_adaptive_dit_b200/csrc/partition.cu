// partition.cu -- PCSP (SAFE-DiT summary, 방법론 2; AccelAes summary B.1):
//   * partition_accumulate: score[i] += sum_h sum_{content j} P[h,i,j] (P in
//     f32 or bf16), one warp per image token, 128-bit streaming loads of the
//     16-byte groups of P that hold a content column (padding is never
//     read), fp64 accumulation and a warp-shuffle reduction;
//   * partition_finalize: the top-k split (ties to the lower index) by an
//     8-pass radix select on order-preserving 64-bit keys (held in shared
//     memory up to 28800 tokens; warp-aggregated histogram), a stable
//     compaction into ascending S / C index lists (a contiguous token range
//     per warp, ballots within it, one scan over the warps), and the
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
// Its inverse (a -0 score comes back as +0, which s treats alike).
__device__ __forceinline__ double key_score(uint64_t key) {
  const uint64_t u = (key >> 63) ? (key & 0x7FFFFFFFFFFFFFFFull) : ~key;
  return __longlong_as_double(static_cast<long long>(u));
}


// Keys kept in shared memory for n up to this many tokens (224 KB, with the
// kernel's static 2 KB under the 227 KB a CTA may hold); larger calls read
// the scores from global memory in every pass.
constexpr int kFinCacheKeys = 28672;

__global__ void __launch_bounds__(kFinThreads, 1)
    finalize_kernel(const double* __restrict__ score, int n, int k, int* __restrict__ idx_s,
                    int* __restrict__ idx_c, float* __restrict__ s_out, int* status) {
  extern __shared__ uint64_t skeys[];  // the n order-preserving keys, when cached
  __shared__ unsigned int hist[256];
  __shared__ int wcount[2][32];        // per warp: keys equal to T, keys selected
  __shared__ int wbase[2][32];         // exclusive prefixes of the same over warps
  __shared__ uint64_t sh_prefix;
  __shared__ int sh_need;
  __shared__ double red_lo[32], red_hi[32];
  __shared__ int sh_nan;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const bool cached = n <= kFinCacheKeys;
  auto key_at = [&](int i) -> uint64_t { return cached ? skeys[i] : score_key(score[i]); };
  if (tid == 0) sh_nan = 0;
  __syncthreads();

  // min / max (exact, order independent), the NaN check, the key cache
  double lo = INFINITY, hi = -INFINITY;
  bool nan_seen = false;
  for (int base = tid; base < n; base += 4 * kFinThreads) {
    double x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * kFinThreads;
      x[u] = i < n ? score[i] : 0.0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * kFinThreads;
      if (i < n) {
        nan_seen |= isnan(x[u]);
        lo = fmin(lo, x[u]);
        hi = fmax(hi, x[u]);
        if (cached) skeys[i] = score_key(x[u]);
      }
    }
  }
  if (nan_seen) sh_nan = 1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    red_lo[wid] = lo;
    red_hi[wid] = hi;
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
    constexpr int U = 4;  // keys of a thread in flight per round
    const int n_up = (n + U * kFinThreads - 1) / (U * kFinThreads) * (U * kFinThreads);
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int b = tid; b < 256; b += kFinThreads) hist[b] = 0;
      __syncthreads();
      for (int base = tid; base < n_up; base += U * kFinThreads) {
        uint64_t kk[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = base + u * kFinThreads;
          kk[u] = i < n ? key_at(i) : 0;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = base + u * kFinThreads;
          const uint32_t bin = (i < n && (kk[u] & pmask) == prefix) ? uint32_t(kk[u] >> shift) & 0xFFu : 256u;
          // one shared-memory atomic per distinct byte in the warp (the keys
          // of a pass share a few leading bytes: per-lane atomics serialise)
          const uint32_t peers = __match_any_sync(0xffffffffu, bin);
          if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], uint32_t(__popc(peers)));
        }
      }
      __syncthreads();
      if (tid < 32) {
        // lane l holds bins 255 - 8 l down to 248 - 8 l (larger keys first)
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          c[e] = hist[255 - 8 * lane - e];
          sum += c[e];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        // the candidates of this pass number at least `remaining`, so some lane hits
        const uint32_t hit = __ballot_sync(0xffffffffu, incl >= uint32_t(remaining));
        if (lane == __ffs(hit) - 1) {
          uint32_t cum = incl - sum;
          int sel = -1;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (sel < 0 && cum + c[e] >= uint32_t(remaining)) sel = 255 - 8 * lane - e;
            if (sel < 0) cum += c[e];
          }
          sh_prefix = prefix | (uint64_t(sel) << shift);
          sh_need = remaining - int(cum);
        }
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

  // stable compaction in token order: warp w owns the contiguous range
  // [w0, w1), walked 32 tokens at a time (coalesced); per-warp counts, one
  // scan over the 32 warps, then every token's place from ballots
  const int per_warp = ((n + 31) / 32 + 31) / 32 * 32;
  const int w0 = min(n, wid * per_warp), w1 = min(n, w0 + per_warp);
  const uint32_t lt = (1u << lane) - 1u;
  auto classify = [&](int i, bool& eq, bool& gt) {
    eq = gt = false;
    if (i >= w1) return;
    if (k >= n) {
      gt = true;
    } else if (k > 0) {
      const uint64_t key = key_at(i);
      eq = key == T;
      gt = key > T;
    }
  };
  int n_eq = 0, n_gt = 0;
  for (int b0 = w0; b0 < w1; b0 += 32) {
    bool eq, gt;
    classify(b0 + lane, eq, gt);
    n_eq += __popc(__ballot_sync(0xffffffffu, eq));
    n_gt += __popc(__ballot_sync(0xffffffffu, gt));
  }
  if (lane == 0) {
    wcount[0][wid] = n_eq;
    wcount[1][wid] = n_gt;
  }
  __syncthreads();
  if (tid < 32) {
    // exclusive scan of the equal counts, then of the selected counts (the
    // keys greater than T, plus the equal ones whose rank is below need_eq)
    const int e = wcount[0][lane];
    int incl = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int eb = incl - e;
    const int sel = wcount[1][lane] + max(0, min(e, need_eq - eb));
    int incl_s = sel;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl_s, o);
      if (lane >= o) incl_s += y;
    }
    wbase[0][lane] = eb;
    wbase[1][lane] = incl_s - sel;
  }
  __syncthreads();
  int eq_rank = wbase[0][wid], pos_s = wbase[1][wid];
  for (int b0 = w0; b0 < w1; b0 += 32) {
    const int i = b0 + lane;
    bool eq, gt;
    classify(i, eq, gt);
    const uint32_t eq_bits = __ballot_sync(0xffffffffu, eq);
    const bool sel = gt || (eq && eq_rank + __popc(eq_bits & lt) < need_eq);
    const uint32_t sel_bits = __ballot_sync(0xffffffffu, sel);
    const int pos = pos_s + __popc(sel_bits & lt);
    if (i < w1) {
      if (sel) {
        if (idx_s && pos < k) idx_s[pos] = i;
      } else {
        if (idx_c && i - pos < n - k) idx_c[i - pos] = i;
      }
      if (s_out) {
        const double x = cached ? key_score(skeys[i]) : score[i];
        s_out[i] = (hi == lo) ? 0.0f : __double2float_rn((x - lo) / (hi - lo));
      }
    }
    eq_rank += __popc(eq_bits);
    pos_s += __popc(sel_bits);
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
  const int cache_bytes = n <= kFinCacheKeys ? n * 8 : 0;
  safedit_status st = set_smem(reinterpret_cast<const void*>(finalize_kernel), kFinCacheKeys * 8);
  if (st != SAFEDIT_OK) return st;
  finalize_kernel<<<1, kFinThreads, cache_bytes, static_cast<cudaStream_t>(stream)>>>(d_score, n, k, d_idx_s,
                                                                                      d_idx_c, d_s, status);
  return after_launch(1);
}

}  // extern "C"
