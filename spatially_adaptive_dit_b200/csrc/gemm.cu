// gemm.cu -- out[r or idx[r], :] = act(A[r, :] W^T + bias) on sm_100a tensor
// cores, the building block of SkipSparse FFN caching (AccelAes summary B.2:
// the FFN runs only on focus tokens, background tokens reuse their cached
// output): the gathered sensitive rows go through W1 (+bias, GELU) and W2
// (+bias), and the second product's rows are scattered into the cached FFN
// state in the epilogue.
//
// Two persistent kernels.  Batches of at least 256 rows run on CTA pairs
// (tcgen05 cta_group::2, 256 x 256 tiles; see gemm_bias_act_pair_kernel).
// Smaller ones run on single CTAs, one 384-thread CTA per SM walking 128 x 256
// output tiles: warp 0 streams A and W k-blocks (64 bf16 wide, 128B swizzle) through
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

// Epilogue of one 128 x 256 accumulator tile by warp `warp` (4..11): the warp
// reads TMEM lanes 32 (warp % 4) .. +31 -- rows row0 + 32 (warp % 4) + lane
// of batch bb, one per thread -- and columns 128 hh .. +127 (hh = (warp - 4) / 4)
// of the tile starting at column n0_tile.  The row destination and the warp's
// 128 bias values are fetched while the accumulator is still being computed.
// `release` hands the warp's part of the accumulator back once it is in
// registers.  Returns false when the wait for the accumulator gave up.
template <class Release>
__device__ __forceinline__ bool epilogue_tile(const GemmParams& p, float* bias_w, uint32_t acc_full,
                                              uint32_t parity, const WaitCtl& ctl, uint32_t acc,
                                              int bb, int row0, int n0_tile, int warp, int lane,
                                              Release release) {
  const int q = warp & 3, hh = (warp - 4) >> 2;
  const int n0 = n0_tile + hh * (kGBN / 2);
  const int r = row0 + q * 32 + lane;
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
  if (!wait_warp(acc_full, parity, ctl)) return false;
  tc_fence_after();
  const int ncols = p.N - n0;  // may be <= 0 for the right half of the last column tile
  __nv_bfloat16* dst = (orow >= 0 && ncols > 0)
                           ? p.out + int64_t(bb) * p.out_bs + int64_t(orow) * p.out_rs + n0
                           : nullptr;
  const uint32_t tl = acc + uint32_t(hh * (kGBN / 2)) + (uint32_t(q * 32) << 16);
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
  if (lane == 0) release();
  emit(vb, 3);
  return true;
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
    float* bias_w = bias_s + (warp - 4) * (kGBN / 2);
    int i = 0;
    for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      const int bm = t / p.tiles_n;
      if (!epilogue_tile(p, bias_w, BAR(ACCF + b), uint32_t((i >> 1) & 1), ctl,
                         tmem + uint32_t(b * kGBN), bm / p.tiles_m, (bm % p.tiles_m) * kGBM,
                         (t % p.tiles_n) * kGBN, warp, lane, [&] { mbar_arrive(BAR(ACCE + b)); }))
        break;
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

// ---------------------------------------------------------------------------
// Pair version (tcgen05 cta_group::2): a cluster of two CTAs on two SMs owns a
// 256 x 256 output tile.  CTA r streams rows 128 r .. +127 of the tile's A
// block and of its W block (half of N) into its own shared memory; one thread
// of CTA 0 issues tcgen05.mma with M = 256, N = 256, which reads A and B from
// both CTAs and writes rows 128 r .. +127 of the accumulator into CTA r's TMEM.
// Each SM thus moves half of the W tile per FLOP of the single-SM kernel.
// Both CTAs' copies complete on CTA 0's stage barriers (cta_group::2 TMA);
// CTA 0's commits arrive on both CTAs' stage-free and accumulator-full
// barriers (multicast commit); both CTAs' epilogue warps hand the accumulator
// back on CTA 0's barrier.  No load is multicast.
constexpr int kG2NS = 6;
constexpr int kG2Stage = 128 * kGBK * 2;  // 16 KB: 128 rows x 64 of A, or of W
constexpr int kG2Smem = 1024 + kG2NS * 2 * kG2Stage + kGBiasBytes + 256;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the variable at shared::cta address `addr` in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(addr), "r"(rank));
  return d;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// 4-D tiled load into this CTA's shared memory, completing on an mbarrier that
// may sit in either CTA of the pair (shared::cluster address)
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const void* tmap, uint32_t bar_cluster,
                                                 int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive once on the barrier at shared::cta offset `bar` of every CTA in
// `mask` when the pair's MMAs issued so far have completed
__device__ __forceinline__ void tc_commit_pair_mc(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// p.tiles_m counts 256-row tiles here; tiles are walked per CTA pair.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
    gemm_bias_act_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmW, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kG2NS * kG2Stage;
  float* bias_s = reinterpret_cast<float*>(smem + kG2NS * 2 * kG2Stage);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kG2NS * 2 * kG2Stage + kGBiasBytes);
  // [0,NS) full (CTA 0's count both CTAs' bytes), [NS,2NS) empty, 2NS+b acc_full[b],
  // 2NS+2+b acc_empty[b] (CTA 0's gets all 16 epilogue warps), 2NS+4 drain
  constexpr int FULL = 0, EMPTY = kG2NS, ACCF = 2 * kG2NS, ACCE = 2 * kG2NS + 2,
                DRAIN = 2 * kG2NS + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + DRAIN + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto BAR = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = int(blockIdx.x >> 1), npairs = int(gridDim.x >> 1);
  const int nk = (p.K + kGBK - 1) / kGBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kG2NS; ++s) {
      mbar_init(BAR(FULL + s), 1);
      mbar_init(BAR(EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(ACCF + b), 1);
      mbar_init(BAR(ACCE + b), 16);
    }
    mbar_init(BAR(DRAIN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512u);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit};

  if (warp == 0) {
    if (lane == 0) {  // TMA producer (both CTAs): this CTA's halves of A and W
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmW);
      int g = 0;
      bool ok = true;
      for (int t = pair; ok && t < p.tiles; t += npairs) {
        const int bm = t / p.tiles_n, n0 = (t % p.tiles_n) * kGBN;
        const int bb = bm / p.tiles_m, m0 = (bm % p.tiles_m) * (2 * kGBM);
        for (int j = 0; j < nk; ++j, ++g) {
          const int s = g % kG2NS;
          if (!(ok = wait_bounded(BAR(EMPTY + s), uint32_t(((g / kG2NS) & 1) ^ 1), ctl))) break;
          if (rank == 0) mbar_arrive_expect_tx(BAR(FULL + s), uint32_t(4 * kG2Stage));
          const uint32_t full0 = mapa_shared(BAR(FULL + s), 0u);
          tma_load_4d_pair(sA + s * kG2Stage, &tmA, full0, j * kGBK, m0 + int(rank) * kGBM, bb, 0);
          tma_load_4d_pair(sB + s * kG2Stage, &tmW, full0, j * kGBK, n0 + int(rank) * kGBM, 0, 0);
        }
      }
      // CTA 0's stage barriers see both CTAs' copies land (already true unless
      // a role aborted before consuming them)
      if (rank == 0)
        for (int j = (g > kG2NS ? g - kG2NS : 0); j < g; ++j)
          wait_drain(BAR(FULL + j % kG2NS), uint32_t((j / kG2NS) & 1), kGDrainNs);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {  // MMA issuer of the pair
      const uint32_t idesc = idesc_bf16_f32(2 * kGBM, kGBN, 0, 0);
      const uint64_t ad0 = smem_desc(sA, 16u, 1024u, 2u), bd0 = smem_desc(sB, 16u, 1024u, 2u);
      auto adv = [](uint64_t d, uint32_t bytes) {
        return (d & 0xFFFFFFFF00000000ull) | uint64_t(uint32_t(d) + (bytes >> 4));
      };
      int g = 0, i = 0;
      bool ok = true;
      for (int t = pair; ok && t < p.tiles; t += npairs, ++i) {
        const int b = i & 1;
        if (!(ok = wait_bounded(BAR(ACCE + b), uint32_t(((i >> 1) & 1) ^ 1), ctl))) break;
        tc_fence_after();
        const uint32_t acc = tmem + uint32_t(b * kGBN);
        for (int j = 0; j < nk; ++j, ++g) {
          const int s = g % kG2NS;
          if (!(ok = wait_bounded(BAR(FULL + s), uint32_t((g / kG2NS) & 1), ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kGBK / 16; ++kk)
            mma_ss_pair(acc, adv(ad0, uint32_t(s * kG2Stage + kk * 32)),
                        adv(bd0, uint32_t(s * kG2Stage + kk * 32)), idesc,
                        (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit_pair_mc(BAR(EMPTY + s), uint16_t(3));
        }
        if (ok) tc_commit_pair_mc(BAR(ACCF + b), uint16_t(3));
      }
      // every MMA of the pair has completed before TMEM is freed, whoever aborted
      tc_commit_pair(BAR(DRAIN));
      wait_drain(BAR(DRAIN), 0u, kGDrainNs);
    }
  } else if (warp >= 4) {
    float* bias_w = bias_s + (warp - 4) * (kGBN / 2);
    int i = 0;
    for (int t = pair; t < p.tiles; t += npairs, ++i) {
      const int b = i & 1;
      const int bm = t / p.tiles_n;
      const uint32_t acce0 = mapa_shared(BAR(ACCE + b), 0u);
      if (!epilogue_tile(p, bias_w, BAR(ACCF + b), uint32_t((i >> 1) & 1), ctl,
                         tmem + uint32_t(b * kGBN), bm / p.tiles_m,
                         (bm % p.tiles_m) * (2 * kGBM) + int(rank) * kGBM, (t % p.tiles_n) * kGBN,
                         warp, lane, [&] { mbar_arrive_remote(acce0); }))
        break;
    }
  }

  // neither CTA frees TMEM or leaves while the pair may still touch it
  tc_fence_before();
  cluster_sync_all();
  if (warp == 2) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512u);
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
  // CTA pairs (256-row tiles) once a batch has at least 256 rows; single CTAs
  // (128-row tiles) below that
  const bool pair = M >= 2 * kGBM;
  const int64_t bm_rows = pair ? 2 * kGBM : kGBM;
  const int64_t tiles_m = (M + bm_rows - 1) / bm_rows, tiles_n = (N + kGBN - 1) / kGBN;
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
  if ((st = make_kmajor_map(&tW, w, uint32_t(pair ? kGBM : kGBN))) != SAFEDIT_OK) return st;
  p.status = status_ptr();
  if (!p.status) return SAFEDIT_ERR_CUDA;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d_idx_out && index_check_enabled() &&
      (st = launch_index_check(d_idx_out, static_cast<int32_t>(M), M_out, p.status, s)) != SAFEDIT_OK)
    return st;
  if (pair) {
    if ((st = set_smem(reinterpret_cast<const void*>(gemm_bias_act_pair_kernel), kG2Smem)) !=
        SAFEDIT_OK)
      return st;
    const int pairs = p.tiles < sms / 2 ? p.tiles : sms / 2;
    gemm_bias_act_pair_kernel<<<2 * pairs, kGThreads, kG2Smem, s>>>(tA, tW, p);
  } else {
    if ((st = set_smem(reinterpret_cast<const void*>(gemm_bias_act_kernel), kGSmem)) != SAFEDIT_OK)
      return st;
    const int grid = p.tiles < sms ? p.tiles : sms;
    gemm_bias_act_kernel<<<grid, kGThreads, kGSmem, s>>>(tA, tW, p);
  }
  return after_launch(1);
}
