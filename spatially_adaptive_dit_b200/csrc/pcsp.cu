// pcsp.cu -- fused PCSP score: image->text cross-attention probabilities and
// their content-weighted aggregation in one pass, without materialising P
// (SAFE-DiT summary, 방법론 2: attention weights from image tokens to text
// content tokens gathered during warm-up; AccelAes summary B.1 step 3).
//
//   score[i] += sum_h  sum_{j valid, content} e_hij / sum_{j valid} e_hij
//
// Persistent CTAs over 128-row tiles; each CTA handles every head of its
// tile, so a row's fp64 sum never leaves the CTA (deterministic, no atomics,
// no scratch).  Per (tile, head) item: TMA brings the Q tile and the text
// block into a 2-stage ring, one tcgen05.mma chain computes S = Q K^T
// (M=128, N = L rounded up to 32) into one of two TMEM accumulators, and the
// two softmax warpgroups (alternate heads) take the row max, then the valid
// and content-weighted exponential sums, two TMEM loads per wait, skipping
// text chunks that are all padding.  Only Q_img is read from HBM.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace sd {

template <int D>
struct PCfg {
  static constexpr int CH = (D % 64 == 0) ? 64 : 32;
  static constexpr int NCH = D / CH;
  static constexpr int ROWB = CH * 2;
  static constexpr uint32_t LAYOUT = (CH == 64) ? 2u : 4u;
  static constexpr int Q_CHUNK = 128 * ROWB;
  static constexpr int Q_BYTES = NCH * Q_CHUNK;
  static constexpr int K_CHUNK = 256 * ROWB;
  static constexpr int K_BYTES = NCH * K_CHUNK;
  static constexpr int STAGE_BYTES = Q_BYTES + K_BYTES;
  static constexpr int NSTAGE = 2;
  static constexpr int TAIL_BYTES = 256 + 2 * 1024 + 1024;  // barriers, vadd, cflag, accs
  static constexpr int USED_BYTES = 1024 + NSTAGE * STAGE_BYTES + TAIL_BYTES;
  // at least 120 KB so that one CTA (holding all 512 TMEM columns) runs per SM
  static constexpr int SMEM_BYTES = USED_BYTES > 120 * 1024 ? USED_BYTES : 120 * 1024;
};

struct PParams {
  const uint8_t* key_valid;  // [L] of the selected batch entry
  const uint8_t* content;    // [L]
  double* score;             // [N]
  int L, Lpad, N, H, b, tiles;
  float scale_log2;
  int* status;
  uint64_t wait_limit;
};

constexpr float kPLog2e = 1.4426950408889634f;
constexpr uint64_t kPDrainNs = 1000000000ull;

template <int D>
__global__ void __launch_bounds__(320, 1)
    pcsp_score_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmKt, const PParams p) {
  using C = PCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sStage = smem_u32(smem);
  uint8_t* tail = smem + C::NSTAGE * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  // bars: [0,2) stage_full, [2,4) stage_empty, [4,6) s_full, [6,8) s_empty,
  //       8 comb (warpgroup 1 partials ready), 9 comb_free, 10 drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 136);
  float* vadd = reinterpret_cast<float*>(tail + 256);          // [256] additive validity
  float* cflag = reinterpret_cast<float*>(tail + 256 + 1024);  // [256] content weight 0/1
  double* accs = reinterpret_cast<double*>(tail + 256 + 2048); // [128] partials of warpgroup 1
  auto BAR = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_units = (p.tiles - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x);
  const int n_items = n_units * p.H;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(0 + i), 1);
      mbar_init(BAR(2 + i), 1);
      mbar_init(BAR(4 + i), 1);
      mbar_init(BAR(6 + i), 128);
    }
    mbar_init(BAR(8), 128);
    mbar_init(BAR(9), 128);
    mbar_init(BAR(10), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int j = tid; j < 256; j += blockDim.x) {
    const bool valid = j < p.L && p.key_valid[j] != 0;
    vadd[j] = valid ? 0.f : -INFINITY;
    cflag[j] = (valid && p.content[j] != 0) ? 1.f : 0.f;
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), 512u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit};

  if (warp < 8) {
    // ============================================= softmax warpgroups
    const int w = warp >> 2, wq = warp & 3, r = tid & 127;
    const uint32_t tl = tmem + uint32_t(w * 256) + (uint32_t(wq * 32) << 16);
    const int nc = p.Lpad / 32;
    uint32_t vmask = 0;  // chunks holding at least one valid key
    for (int c = 0; c < nc; ++c) {
      bool any = false;
      for (int e = 0; e < 32; ++e) any |= (vadd[c * 32 + e] == 0.f);
      if (any) vmask |= 1u << c;
    }
    const float sl2 = p.scale_log2;
    int cnt = 0;  // items processed by this warpgroup (TMEM buffer phase)
    bool ok = true;
    for (int i = 0; i < n_units && ok; ++i) {
      const int tile = int(blockIdx.x) + i * int(gridDim.x);
      const int row = tile * 128 + r;
      double acc = 0.0;
      for (int h = 0; h < p.H; ++h) {
        const int n = i * p.H + h;
        if ((n & 1) != w) continue;
        if (!(ok = wait_warp(BAR(4 + w), uint32_t(cnt & 1), ctl))) break;
        ++cnt;
        tc_fence_after();
        float m = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < nc; c += 2) {
          const bool a = (vmask >> c) & 1u, b2 = (c + 1 < nc) && ((vmask >> (c + 1)) & 1u);
          if (!a && !b2) continue;
          uint32_t v0[32], v1[32];
          tmem_ld32(tl + uint32_t(c * 32), v0);
          tmem_ld32(tl + uint32_t((c + 1) * 32), v1);
          tmem_wait_ld();
          if (a) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              m = fmaxf(m, fmaf(__uint_as_float(v0[e]), sl2, vadd[c * 32 + e]));
          }
          if (b2) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              m = fmaxf(m, fmaf(__uint_as_float(v1[e]), sl2, vadd[(c + 1) * 32 + e]));
          }
        }
        const float m_use = (m == -INFINITY) ? 0.f : m;
        float sv[4] = {0.f, 0.f, 0.f, 0.f}, sc[4] = {0.f, 0.f, 0.f, 0.f};
        int last = -1;
        for (int c = 0; c < nc; ++c)
          if ((vmask >> c) & 1u) last = c;
#pragma unroll 1
        for (int c = 0; c < nc; c += 2) {
          const bool a = (vmask >> c) & 1u, b2 = (c + 1 < nc) && ((vmask >> (c + 1)) & 1u);
          if (!a && !b2) continue;
          uint32_t v0[32], v1[32];
          tmem_ld32(tl + uint32_t(c * 32), v0);
          tmem_ld32(tl + uint32_t((c + 1) * 32), v1);
          tmem_wait_ld();
          if (c + 1 >= last) {  // last TMEM read of this accumulator
            tc_fence_before();
            mbar_arrive(BAR(6 + w));
          }
          if (a) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int j = c * 32 + e;
              const float ev = ex2_approx(fmaf(__uint_as_float(v0[e]), sl2, vadd[j]) - m_use);
              sv[e & 3] += ev;
              sc[e & 3] = fmaf(ev, cflag[j], sc[e & 3]);
            }
          }
          if (b2) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int j = (c + 1) * 32 + e;
              const float ev = ex2_approx(fmaf(__uint_as_float(v1[e]), sl2, vadd[j]) - m_use);
              sv[e & 3] += ev;
              sc[e & 3] = fmaf(ev, cflag[j], sc[e & 3]);
            }
          }
        }
        if (last < 0) {  // no valid key at all: nothing was read
          tc_fence_before();
          mbar_arrive(BAR(6 + w));
        }
        const float tv = (sv[0] + sv[1]) + (sv[2] + sv[3]);
        const float tcn = (sc[0] + sc[1]) + (sc[2] + sc[3]);
        if (tv > 0.f)
          acc += static_cast<double>(tcn) / static_cast<double>(tv);
        else if (row < p.N)
          set_status(p.status, SAFEDIT_ERR_MASKED_ROW);
      }
      if (!ok) break;
      // combine the two warpgroups' partial sums of this tile (fixed order)
      if (w == 1) {
        if (i > 0 && !(ok = wait_warp(BAR(9), uint32_t((i - 1) & 1), ctl))) break;
        accs[r] = acc;
        mbar_arrive(BAR(8));
      } else {
        if (!(ok = wait_warp(BAR(8), uint32_t(i & 1), ctl))) break;
        const double total = acc + accs[r];
        mbar_arrive(BAR(9));
        if (row < p.N) p.score[row] += total;
      }
    }
  } else if (warp == 8) {
    // ============================================= TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmKt);
      int issued = 0;
      for (int n = 0; n < n_items; ++n) {
        const int st = n & 1;
        if (!wait_bounded(BAR(2 + st), uint32_t(((n >> 1) & 1) ^ 1), ctl)) break;
        const int i = n / p.H, h = n - i * p.H;
        const int tile = int(blockIdx.x) + i * int(gridDim.x);
        const uint32_t sQ = sStage + uint32_t(st * C::STAGE_BYTES), sK = sQ + C::Q_BYTES;
        mbar_arrive_expect_tx(BAR(0 + st), uint32_t(C::Q_BYTES + C::NCH * p.Lpad * C::ROWB));
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          tma_load_4d(sQ + c * C::Q_CHUNK, &tmQ, BAR(0 + st), c * C::CH, tile * 128, h, p.b);
          tma_load_4d(sK + c * C::K_CHUNK, &tmKt, BAR(0 + st), c * C::CH, 0, h, p.b);
        }
        issued = n + 1;
      }
      // every copy has landed before the CTA leaves (already true unless a
      // role aborted before consuming it)
      for (int n = (issued > 2 ? issued - 2 : 0); n < issued; ++n)
        wait_drain(BAR(0 + (n & 1)), uint32_t((n >> 1) & 1), kPDrainNs);
    }
  } else {
    // ============================================= MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, p.Lpad, 0, 0);
      constexpr uint32_t SBO = 8u * C::ROWB;
      bool ok = true;
      for (int n = 0; n < n_items && ok; ++n) {
        const int st = n & 1;
        if (!(ok = wait_bounded(BAR(0 + st), uint32_t((n >> 1) & 1), ctl))) break;
        if (!(ok = wait_bounded(BAR(6 + st), uint32_t(((n >> 1) & 1) ^ 1), ctl))) break;
        tc_fence_after();
        const uint32_t sQ = sStage + uint32_t(st * C::STAGE_BYTES), sK = sQ + C::Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int chunk = (kk * 16) / C::CH;
          const uint32_t within = uint32_t(((kk * 16) % C::CH) * 2);
          mma_ss(tmem + uint32_t(st * 256),
                 smem_desc(sQ + chunk * C::Q_CHUNK + within, 16u, SBO, C::LAYOUT),
                 smem_desc(sK + chunk * C::K_CHUNK + within, 16u, SBO, C::LAYOUT), idesc,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(BAR(4 + st));
        tc_commit(BAR(2 + st));
      }
      // every MMA has completed before TMEM is freed, whoever aborted
      tc_commit(BAR(10));
      wait_drain(BAR(10), 0u, kPDrainNs);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512u);
  }
}

template <int D>
static safedit_status launch_p(const CUtensorMap& q, const CUtensorMap& k, const PParams& p,
                               cudaStream_t s) {
  auto kern = pcsp_score_kernel<D>;
  safedit_status st = set_smem(reinterpret_cast<const void*>(kern), PCfg<D>::SMEM_BYTES);
  if (st != SAFEDIT_OK) return st;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.tiles < sms ? p.tiles : sms;
  kern<<<grid, 320, PCfg<D>::SMEM_BYTES, s>>>(q, k, p);
  return after_launch(1);
}

}  // namespace sd

using namespace sd;

extern "C" safedit_status safedit_pcsp_score(const safedit_tensor* q_img, const safedit_tensor* k_txt,
                                             const uint8_t* d_key_valid, const uint8_t* d_content,
                                             int32_t batch_index, float scale, double* d_score,
                                             void* stream) {
  safedit_status st;
  for (const safedit_tensor* t : {q_img, k_txt}) {
    if ((st = check_tensor(t, 4)) != SAFEDIT_OK) return st;
    if (t->dtype != SAFEDIT_BF16) return SAFEDIT_ERR_DTYPE;
    if (t->strides[3] != 1 || !aligned16(t->data)) return SAFEDIT_ERR_ALIGNMENT;
    for (int i = 0; i < 3; ++i)
      if (t->strides[i] % 8 != 0 || t->strides[i] < 0) return SAFEDIT_ERR_ALIGNMENT;
  }
  if (!d_key_valid || !d_content) return SAFEDIT_ERR_INVALID_ARG;
  const int64_t B = q_img->dims[0], H = q_img->dims[1], N = q_img->dims[2], D = q_img->dims[3];
  if (N > 0 && !d_score) return SAFEDIT_ERR_INVALID_ARG;
  const int64_t L = k_txt->dims[2];
  if (k_txt->dims[0] != B || k_txt->dims[1] != H || k_txt->dims[3] != D) return SAFEDIT_ERR_SHAPE;
  if (batch_index < 0 || batch_index >= B) return SAFEDIT_ERR_INVALID_ARG;
  if (D != 64 && D != 96 && D != 128) return SAFEDIT_ERR_UNSUPPORTED;
  if (L < 1 || L > 256) return SAFEDIT_ERR_UNSUPPORTED;
  if (N == 0 || H == 0) return SAFEDIT_OK;
  if (N > INT32_MAX - 128 || H > 65535) return SAFEDIT_ERR_SHAPE;
  PParams p{};
  p.key_valid = d_key_valid + int64_t(batch_index) * L;
  p.content = d_content;
  p.score = d_score;
  p.L = static_cast<int>(L);
  p.Lpad = static_cast<int>((L + 31) / 32 * 32);
  p.N = static_cast<int>(N);
  p.H = static_cast<int>(H);
  p.b = batch_index;
  p.tiles = static_cast<int>((N + 127) / 128);
  const float sc = (scale > 0.f) ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale_log2 = sc * kPLog2e;
  p.wait_limit = wait_limit_ns();
  const int ch = (D % 64 == 0) ? 64 : 32;
  const CUtensorMapSwizzle swz = ch == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap tq, tk;
  {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(N), uint64_t(H), uint64_t(B)};
    const uint64_t str[3] = {uint64_t(q_img->strides[2]) * 2, uint64_t(q_img->strides[1]) * 2,
                             uint64_t(q_img->strides[0]) * 2};
    const uint32_t box[4] = {uint32_t(ch), 128u, 1u, 1u};
    if ((st = encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, q_img->data, dims, str, box,
                          swz)) != SAFEDIT_OK)
      return st;
  }
  {
    const uint64_t dims[4] = {uint64_t(D), uint64_t(L), uint64_t(H), uint64_t(B)};
    const uint64_t str[3] = {uint64_t(k_txt->strides[2]) * 2, uint64_t(k_txt->strides[1]) * 2,
                             uint64_t(k_txt->strides[0]) * 2};
    const uint32_t box[4] = {uint32_t(ch), uint32_t(p.Lpad), 1u, 1u};
    if ((st = encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, k_txt->data, dims, str, box,
                          swz)) != SAFEDIT_OK)
      return st;
  }
  p.status = status_ptr();
  if (!p.status) return SAFEDIT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (D) {
    case 64: return launch_p<64>(tq, tk, p, s);
    case 96: return launch_p<96>(tq, tk, p, s);
    default: return launch_p<128>(tq, tk, p, s);
  }
}
