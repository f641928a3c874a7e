// gemm.cu -- out[r or idx[r], :] = act(A[r, :] W^T + bias) on sm_100a tensor
// cores, the building block of SkipSparse FFN caching (AccelAes summary B.2:
// the FFN runs only on focus tokens, background tokens reuse their cached
// output): the gathered sensitive rows go through W1 (+bias, GELU) and W2
// (+bias), and the second product's rows are scattered into the cached FFN
// state in the epilogue.
//
// Persistent kernel, one 384-thread CTA per SM walking 128 x 256 output
// tiles: warp 0 streams A and W k-blocks (64 bf16 wide, 128B swizzle) through
// a 4-stage TMA ring, warp 1 issues tcgen05.mma (M=128, N=256, K=16) into one
// of two 256-column fp32 TMEM accumulators, warps 4-11 (thread = output row =
// TMEM lane, two warps per row quarter, 128 columns each) drain the other
// accumulator meanwhile: TMEM -> registers, bias, GELU (tanh form), bf16,
// 16-byte stores to the row's destination.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace sd {

constexpr int kGBM = 128, kGBN = 256, kGBK = 64, kGNS = 4;
constexpr int kGAStage = kGBM * kGBK * 2;  // 16 KB
constexpr int kGBStage = kGBN * kGBK * 2;  // 32 KB
constexpr int kGBiasBytes = 8 * (kGBN / 2) * 4;  // 128 bias values per epilogue warp
constexpr int kGSmem = 1024 + kGNS * (kGAStage + kGBStage) + kGBiasBytes + 256;
constexpr int kGThreads = 384;
constexpr uint64_t kGDrainNs = 1000000000ull;

struct GemmParams {
  const float* bias;  // nullable [N]
  __nv_bfloat16* out;
  int64_t out_rs, out_bs;  // row / batch strides (elements)
  const int* idx;          // nullable: output row of A row r is idx[r] (every batch)
  int M, N, K, M_out, act;
  // row tiles per batch, column tiles, all tiles (B x tiles_m x tiles_n).  The
  // column index runs fastest, so the CTAs in flight share a few row blocks
  // of A and sweep all of W: W stays in L2 and A is read from HBM once.
  int tiles_m, tiles_n, tiles;
  int* status;
  uint64_t wait_limit;
};

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// GELU, tanh form (Hendrycks & Gimpel): 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
__device__ __forceinline__ float gelu_tanh(float x) {
  const float c = 0.7978845608028654f;
  const float u = c * fmaf(0.044715f * x, x * x, x);
  return 0.5f * x * (1.f + tanh_approx(u));
}

// tcgen05.wait::ld, then an empty asm that redefines the loaded registers,
// so that no use of them can be scheduled above the wait
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&v)[32]) {
  tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < 32; ++e) asm volatile("" : "+r"(v[e]));
}

__global__ void __launch_bounds__(kGThreads, 1)
    gemm_bias_act_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmW, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kGNS * kGAStage;
  float* bias_s = reinterpret_cast<float*>(smem + kGNS * (kGAStage + kGBStage));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGNS * (kGAStage + kGBStage) + kGBiasBytes);
  // [0,NS) full, [NS,2NS) empty, 2NS+b acc_full[b], 2NS+2+b acc_empty[b], 2NS+4 drain
  constexpr int FULL = 0, EMPTY = kGNS, ACCF = 2 * kGNS, ACCE = 2 * kGNS + 2, DRAIN = 2 * kGNS + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + DRAIN + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto BAR = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (p.K + kGBK - 1) / kGBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGNS; ++s) {
      mbar_init(BAR(FULL + s), 1);
      mbar_init(BAR(EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(ACCF + b), 1);
      mbar_init(BAR(ACCE + b), 8);
    }
    mbar_init(BAR(DRAIN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit};

  if (warp == 0) {
    if (lane == 0) {  // TMA producer: one ring over every tile's k-blocks
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmW);
      int g = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
        const int bm = t / p.tiles_n, n0 = (t % p.tiles_n) * kGBN;
        const int bb = bm / p.tiles_m, m0 = (bm % p.tiles_m) * kGBM;
        for (int j = 0; j < nk; ++j, ++g) {
          const int s = g % kGNS;
          if (!(ok = wait_bounded(BAR(EMPTY + s), uint32_t(((g / kGNS) & 1) ^ 1), ctl))) break;
          mbar_arrive_expect_tx(BAR(FULL + s), uint32_t(kGAStage + kGBStage));
          tma_load_4d(sA + s * kGAStage, &tmA, BAR(FULL + s), j * kGBK, m0, bb, 0);
          tma_load_4d(sB + s * kGBStage, &tmW, BAR(FULL + s), j * kGBK, n0, 0, 0);
        }
      }
      // every copy has landed before the CTA leaves (already true unless a
      // role aborted before consuming it)
      for (int j = (g > kGNS ? g - kGNS : 0); j < g; ++j)
        wait_drain(BAR(FULL + j % kGNS), uint32_t((j / kGNS) & 1), kGDrainNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kGBM, kGBN, 0, 0);
      const uint64_t ad0 = smem_desc(sA, 16u, 1024u, 2u), bd0 = smem_desc(sB, 16u, 1024u, 2u);
      auto adv = [](uint64_t d, uint32_t bytes) {
        return (d & 0xFFFFFFFF00000000ull) | uint64_t(uint32_t(d) + (bytes >> 4));
      };
      int g = 0, i = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++i) {
        const int b = i & 1;
        if (!(ok = wait_bounded(BAR(ACCE + b), uint32_t(((i >> 1) & 1) ^ 1), ctl))) break;
        tc_fence_after();
        const uint32_t acc = tmem + uint32_t(b * kGBN);
        for (int j = 0; j < nk; ++j, ++g) {
          const int s = g % kGNS;
          if (!(ok = wait_bounded(BAR(FULL + s), uint32_t((g / kGNS) & 1), ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kGBK / 16; ++kk)
            mma_ss(acc, adv(ad0, uint32_t(s * kGAStage + kk * 32)),
                   adv(bd0, uint32_t(s * kGBStage + kk * 32)), idesc, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(BAR(EMPTY + s));
        }
        if (ok) tc_commit(BAR(ACCF + b));
      }
      // every MMA has completed before TMEM is freed, whoever aborted
      tc_commit(BAR(DRAIN));
      wait_drain(BAR(DRAIN), 0u, kGDrainNs);
    }
  } else if (warp >= 4) {
    // epilogue, warps 4-11: warp w reads TMEM lanes 32 (w % 4) .. +31 (its
    // 32 tile rows, one per thread) and columns 128 hh .. +127 of the tile
    const int q = warp & 3, hh = (warp - 4) >> 2;
    float* bias_w = bias_s + (warp - 4) * (kGBN / 2);
    int i = 0;
    for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      const int bm = t / p.tiles_n, n0 = (t % p.tiles_n) * kGBN + hh * (kGBN / 2);
      const int bb = bm / p.tiles_m, r = (bm % p.tiles_m) * kGBM + q * 32 + lane;
      // row destination and this warp's 128 bias values, fetched while the
      // accumulator is still being computed
      int orow = r < p.M ? r : -1;
      if (orow >= 0 && p.idx) {
        orow = __ldg(p.idx + r);
        if (orow < 0 || orow >= p.M_out) {
          set_status(p.status, SAFEDIT_ERR_INDEX);
          orow = -1;
        }
      }
      __syncwarp();  // the previous tile's reads of bias_w are done
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = n0 + lane * 4 + e;
        bias_w[lane * 4 + e] = (p.bias && n < p.N) ? __ldg(p.bias + n) : 0.f;
      }
      __syncwarp();
      if (!wait_warp(BAR(ACCF + b), uint32_t((i >> 1) & 1), ctl)) break;
      tc_fence_after();
      const int ncols = p.N - n0;  // may be <= 0 for the right half of the last column tile
      __nv_bfloat16* dst = (orow >= 0 && ncols > 0)
                               ? p.out + int64_t(bb) * p.out_bs + int64_t(orow) * p.out_rs + n0
                               : nullptr;
      const uint32_t tl =
          tmem + uint32_t(b * kGBN + hh * (kGBN / 2)) + (uint32_t(q * 32) << 16);
      auto emit = [&](const uint32_t (&v)[32], int c) {
        if (!dst || c * 32 >= ncols) return;
        const float4* bv = reinterpret_cast<const float4*>(bias_w + c * 32);
        uint32_t w[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 bz = bv[e4];
          float x[4] = {__uint_as_float(v[4 * e4]) + bz.x, __uint_as_float(v[4 * e4 + 1]) + bz.y,
                        __uint_as_float(v[4 * e4 + 2]) + bz.z, __uint_as_float(v[4 * e4 + 3]) + bz.w};
          if (p.act == 1) {
#pragma unroll
            for (int z = 0; z < 4; ++z) x[z] = gelu_tanh(x[z]);
          }
          w[2 * e4] = pack_bf16x2(x[0], x[1]);
          w[2 * e4 + 1] = pack_bf16x2(x[2], x[3]);
        }
        // N is a multiple of 8, so a 32-column chunk is whole 16-byte units
        uint4* o4 = reinterpret_cast<uint4*>(dst + c * 32);
        const int units = min(4, (ncols - c * 32) >> 3);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (e < units) o4[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
      };
      // four 32-column chunks, the TMEM load of the next overlapping the math of this one
      uint32_t va[32], vb[32];
      tmem_ld32(tl, va);
      tmem_wait_ld_regs(va);
      tmem_ld32(tl + 32u, vb);
      emit(va, 0);
      tmem_wait_ld_regs(vb);
      tmem_ld32(tl + 64u, va);
      emit(vb, 1);
      tmem_wait_ld_regs(va);
      tmem_ld32(tl + 96u, vb);
      emit(va, 2);
      tmem_wait_ld_regs(vb);
      // this warp's part of the accumulator is in registers: hand it back
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(ACCE + b));
      emit(vb, 3);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512u);
  }
}

// K-major bf16 operand [B, rows, K] (B = 1 for 2-D) as a 4-D map {K, rows,
// B, 1}, box {64, box_rows, 1, 1}, 128-byte swizzle.
static safedit_status make_kmajor_map(CUtensorMap* m, const safedit_tensor* t, uint32_t box_rows) {
  const int r = t->ndim;
  const int64_t rows = t->dims[r - 2], K = t->dims[r - 1], B = r == 3 ? t->dims[0] : 1;
  const int64_t rs = t->strides[r - 2], bs = r == 3 ? t->strides[0] : rows * rs;
  const uint64_t dims[4] = {uint64_t(K), uint64_t(rows), uint64_t(B), 1u};
  const uint64_t strides[3] = {uint64_t(rs) * 2, uint64_t(bs) * 2, uint64_t(bs) * B * 2};
  const uint32_t box[4] = {uint32_t(kGBK), box_rows, 1u, 1u};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace sd

using namespace sd;

extern "C" safedit_status safedit_gemm_bias_act(const safedit_tensor* a, const safedit_tensor* w,
                                                const float* d_bias, int32_t act,
                                                const int32_t* d_idx_out,
                                                const safedit_tensor* out, void* stream) {
  if (!a || !w || !out) return SAFEDIT_ERR_INVALID_ARG;
  const int rank = a->ndim;
  if (rank != 2 && rank != 3) return SAFEDIT_ERR_SHAPE;
  safedit_status st;
  if ((st = check_tensor(a, rank)) != SAFEDIT_OK) return st;
  if ((st = check_tensor(w, 2)) != SAFEDIT_OK) return st;
  if ((st = check_tensor(out, rank)) != SAFEDIT_OK) return st;
  for (const safedit_tensor* t : {a, w, out})
    if (t->dtype != SAFEDIT_BF16) return SAFEDIT_ERR_DTYPE;
  const int64_t B = rank == 3 ? a->dims[0] : 1;
  const int64_t M = a->dims[rank - 2], K = a->dims[rank - 1], N = w->dims[0];
  const int64_t M_out = out->dims[rank - 2];
  if (w->dims[1] != K || out->dims[rank - 1] != N) return SAFEDIT_ERR_SHAPE;
  if (rank == 3 && out->dims[0] != B) return SAFEDIT_ERR_SHAPE;
  if (!d_idx_out && M_out != M) return SAFEDIT_ERR_SHAPE;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX || M_out > INT32_MAX) return SAFEDIT_ERR_SHAPE;
  if (act != 0 && act != 1) return SAFEDIT_ERR_INVALID_ARG;
  if (N % 8 != 0) return SAFEDIT_ERR_ALIGNMENT;  // whole 16-byte output units
  if (M == 0 || N == 0 || B == 0) return SAFEDIT_OK;  // strides of empty tensors are not checked
  if (K == 0) return SAFEDIT_ERR_SHAPE;
  for (const safedit_tensor* t : {a, w, out}) {
    const int r = t->ndim;
    if (t->strides[r - 1] != 1 || t->strides[r - 2] <= 0 || t->strides[r - 2] % 8 != 0 ||
        !aligned16(t->data))
      return SAFEDIT_ERR_ALIGNMENT;
    if (r == 3 && (t->strides[0] <= 0 || t->strides[0] % 8 != 0)) return SAFEDIT_ERR_ALIGNMENT;
  }
  const int64_t tiles_m = (M + kGBM - 1) / kGBM, tiles_n = (N + kGBN - 1) / kGBN;
  const int64_t tiles = tiles_m * B * tiles_n;
  if (tiles > INT32_MAX) return SAFEDIT_ERR_SHAPE;
  GemmParams p{};
  p.bias = d_bias;
  p.out = static_cast<__nv_bfloat16*>(out->data);
  p.out_rs = out->strides[rank - 2];
  p.out_bs = rank == 3 ? out->strides[0] : 0;
  p.idx = d_idx_out;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.M_out = static_cast<int>(M_out);
  p.act = act;
  p.tiles_m = static_cast<int>(tiles_m);
  p.tiles_n = static_cast<int>(tiles_n);
  p.tiles = static_cast<int>(tiles);
  p.wait_limit = wait_limit_ns();
  CUtensorMap tA, tW;
  if ((st = make_kmajor_map(&tA, a, uint32_t(kGBM))) != SAFEDIT_OK) return st;
  if ((st = make_kmajor_map(&tW, w, uint32_t(kGBN))) != SAFEDIT_OK) return st;
  p.status = status_ptr();
  if (!p.status) return SAFEDIT_ERR_CUDA;
  if ((st = set_smem(reinterpret_cast<const void*>(gemm_bias_act_kernel), kGSmem)) != SAFEDIT_OK)
    return st;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.tiles < sms ? p.tiles : sms;
  gemm_bias_act_kernel<<<grid, kGThreads, kGSmem, static_cast<cudaStream_t>(stream)>>>(tA, tW, p);
  return after_launch(1);
}
