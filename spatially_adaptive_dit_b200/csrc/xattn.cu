// xattn.cu -- PCSP score producer: image->text cross-attention probabilities
// for one batch entry (SAFE-DiT summary, 방법론 2: attention weights from
// image tokens to text tokens gathered during warm-up; AccelAes summary B.1
// step 3).  Text padding is a kept semantic mask (방법론 1 보존): padding keys
// receive exactly 0.
//
// Persistent: one 320-thread CTA per SM over (head, 128-row tile) units.  TMA
// brings the Q tile and the whole text-key block (L <= 256, reloaded only on a
// head change) into swizzled shared memory; one elected thread issues
// tcgen05.mma for S = Q K^T (M=128, N=L rounded up to 32) into one of two
// 256-column TMEM accumulators; two softmax warpgroups (thread = row = TMEM
// lane) take alternate units and run three TMEM passes (max; exp + sum with
// the exponentials written back to TMEM; scale).  The probabilities leave
// through 4-deep 128B-swizzled shared-memory staging per warpgroup and TMA
// tensor stores, so the 4-byte P writes reach HBM as full lines; text chunks
// that are all padding skip TMEM and the exponential unit and are stored from
// one shared all-zero box.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace sd {

template <int D>
struct XCfg {
  static constexpr int CH = (D % 64 == 0) ? 64 : 32;
  static constexpr int NCH = D / CH;
  static constexpr int ROWB = CH * 2;
  static constexpr uint32_t LAYOUT = (CH == 64) ? 2u : 4u;
  static constexpr int Q_CHUNK = 128 * ROWB;
  static constexpr int Q_BYTES = NCH * Q_CHUNK;
  static constexpr int K_CHUNK = 256 * ROWB;  // room for L <= 256 rows
  static constexpr int K_BYTES = NCH * K_CHUNK;
  static constexpr int STAGE_BYTES = Q_BYTES + K_BYTES;  // one Q tile + one text block
  // One load stage: the next unit's loads still overlap the current unit's
  // softmax (the MMA frees the stage long before the softmax ends); the smem
  // goes to staging so that more TMA stores stay in flight.
  static constexpr int NSTAGE = 1;
  static constexpr int NOUT = (D == 128) ? 3 : 4;      // staging buffers per warpgroup
  static constexpr int OUT_BYTES = 128 * 128;          // 128 rows x 32 f32
  // + one all-zero box that every all-padding chunk is stored from
  static constexpr int SMEM_BYTES =
      1024 + NSTAGE * STAGE_BYTES + (2 * NOUT + 1) * OUT_BYTES + 256 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct XParams {
  const uint8_t* key_valid;  // [L] of the selected batch entry
  float* P;                  // [H,N,L] output (for the L % 4 tail columns)
  int64_t p_sh, p_sn;        // element strides of P
  int L, L4, Lpad, N, H, b;  // L4 = L rounded down to 4: the TMA-stored columns
  int tiles;                 // 128-row tiles per head
  int units;                 // H * tiles
  float scale_log2;
  int* status;
  uint64_t wait_limit;
};

constexpr float kXLog2e = 1.4426950408889634f;
constexpr uint64_t kXDrainNs = 1000000000ull;

// Persistent: CTA c owns a contiguous range of (head, 128-row tile) units.
// Warps 0-3 and 4-7: two softmax warpgroups taking alternate units, each on
// its own 256-column TMEM accumulator; warp 8: TMA producer; warp 9: MMA.
template <int D>
__global__ void __launch_bounds__(320, 1)
    xattn_probs_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmKt,
                       const __grid_constant__ CUtensorMap tmP, const XParams p) {
  using C = XCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sStage = smem_u32(smem);
  const uint32_t sOut = sStage + C::NSTAGE * C::STAGE_BYTES;  // 2 x NOUT staging buffers
  const uint32_t sZero = sOut + 2 * C::NOUT * C::OUT_BYTES;   // zeros, never rewritten
  uint8_t* tail = smem + C::NSTAGE * C::STAGE_BYTES + (2 * C::NOUT + 1) * C::OUT_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tail);
  // bars: [0,2) stage_full, [2,4) stage_empty, [4,6) s_full, [6,8) s_empty, 8 drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + 96);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 104);
  float* vadd = reinterpret_cast<float*>(tail + 256);  // [256] additive validity
  auto BAR = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int per = p.units / int(gridDim.x), extra = p.units % int(gridDim.x);
  const int u0 = int(blockIdx.x) * per + min(int(blockIdx.x), extra);
  const int n_local = per + (int(blockIdx.x) < extra ? 1 : 0);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(0 + i), 1);
      mbar_init(BAR(2 + i), 1);
      mbar_init(BAR(4 + i), 1);
      mbar_init(BAR(6 + i), 128);
    }
    mbar_init(BAR(8), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int j = tid; j < 256; j += blockDim.x)
    vadd[j] = (j < p.L && p.key_valid[j] != 0) ? 0.f : -INFINITY;
  for (int j = tid; j < C::OUT_BYTES / 16; j += blockDim.x)
    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(sZero + 16u * uint32_t(j)), "r"(0u)
                 : "memory");
  fence_proxy_async_smem();  // the zero box is read by TMA stores
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
    const int nc = p.Lpad / 32;  // 32-column chunks (Lpad is a multiple of 32)
    // chunks with at least one valid key; all-padding chunks are written as
    // zeros without touching TMEM or the exponential unit
    uint32_t vmask = 0;
    for (int c = 0; c < nc; ++c) {
      bool any = false;
      for (int e = 0; e < 32; ++e) any |= (vadd[c * 32 + e] == 0.f);
      if (any) vmask |= 1u << c;
    }
    const float sl2 = p.scale_log2;
    int nstore = 0;  // TMA stores issued by this warpgroup (staging buffer = nstore % NOUT)
    for (int i = w; i < n_local; i += 2) {
      const int u = u0 + i, h = u / p.tiles, tile = u - h * p.tiles;
      const int row0 = tile * 128;
      if (!wait_warp(BAR(4 + w), uint32_t((i >> 1) & 1), ctl)) break;
      tc_fence_after();
      // pass 1: row max over valid keys
      float m = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < nc; c += 2) {
        const bool a = (vmask >> c) & 1u, b2 = (c + 1 < nc) && ((vmask >> (c + 1)) & 1u);
        if (!a && !b2) continue;
        uint32_t v0[32], v1[32];
        // both chunks are loaded (a pair never leaves the 256-column accumulator)
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
      // pass 2: exponentials (written back to TMEM) and their sum
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll 1
      for (int c = 0; c < nc; c += 2) {
        const bool a = (vmask >> c) & 1u, b2 = (c + 1 < nc) && ((vmask >> (c + 1)) & 1u);
        if (!a && !b2) continue;
        uint32_t v0[32], v1[32];
        // both chunks are loaded (a pair never leaves the 256-column accumulator)
        tmem_ld32(tl + uint32_t(c * 32), v0);
        tmem_ld32(tl + uint32_t((c + 1) * 32), v1);
        tmem_wait_ld();
        if (a) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float ev = ex2_approx(fmaf(__uint_as_float(v0[e]), sl2, vadd[c * 32 + e]) - m_use);
            sum0 += ev;
            v0[e] = __float_as_uint(ev);
          }
          tmem_st32(tl + uint32_t(c * 32), v0);
        }
        if (b2) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float ev =
                ex2_approx(fmaf(__uint_as_float(v1[e]), sl2, vadd[(c + 1) * 32 + e]) - m_use);
            sum1 += ev;
            v1[e] = __float_as_uint(ev);
          }
          tmem_st32(tl + uint32_t((c + 1) * 32), v1);
        }
      }
      tmem_wait_st();
      const float sum = sum0 + sum1;
      if (!(sum > 0.f) && row0 + r < p.N) set_status(p.status, SAFEDIT_ERR_MASKED_ROW);
      const float inv = (sum > 0.f) ? 1.f / sum : 0.f;
      // pass 3: normalise, stage (128B swizzle) and store 128 x 32 boxes
      int last_valid = -1;
      for (int c = 0; c < nc; ++c)
        if ((vmask >> c) & 1u) last_valid = c;
      if (last_valid < 0) {  // no TMEM read in this pass: the accumulator is free now
        tc_fence_before();
        mbar_arrive(BAR(6 + w));
      }
      // all-padding chunks first: stored from the zero box, no staging, so
      // that those writes overlap the normalise pass below
      if (r == 0) {
        for (int c = 0; c < nc; ++c)
          if (!((vmask >> c) & 1u) && c * 32 < p.L4) {
            tma_store_3d(&tmP, sZero, c * 32, row0, h);
            bulk_commit();
          }
      }
#pragma unroll 1
      for (int c = 0; c < nc; ++c) {
        if (!((vmask >> c) & 1u)) {
          if (p.L4 < p.L && row0 + r < p.N) {
            for (int j = max(c * 32, p.L4); j < min(c * 32 + 32, p.L); ++j)
              p.P[h * p.p_sh + int64_t(row0 + r) * p.p_sn + j] = 0.f;
          }
          continue;
        }
        uint32_t v[32];
        tmem_ld32(tl + uint32_t(c * 32), v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * inv);
        if (c == last_valid) {  // the accumulator is free for the next unit
          tc_fence_before();
          mbar_arrive(BAR(6 + w));
        }
        const uint32_t buf = sOut + uint32_t((w * C::NOUT + (nstore % C::NOUT)) * C::OUT_BYTES);
        if (nstore >= C::NOUT) {
          if (r == 0) bulk_wait_read<C::NOUT - 1>();
          named_bar_sync(1 + w, 128);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t off = uint32_t(r * 128 + ((q ^ (r & 7)) * 16));
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + off), "r"(v[4 * q]),
                       "r"(v[4 * q + 1]), "r"(v[4 * q + 2]), "r"(v[4 * q + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
        named_bar_sync(1 + w, 128);
        if (c * 32 < p.L4) {
          // the tensor map spans the first L4 columns: TMA stores move whole
          // 16-byte units, so the last L % 4 columns are written below instead
          if (r == 0) {
            tma_store_3d(&tmP, buf, c * 32, row0, h);
            bulk_commit();
          }
          ++nstore;
        }
        if (p.L4 < p.L && row0 + r < p.N) {
          for (int e = 0; e < 32; ++e) {
            const int j = c * 32 + e;
            if (j >= p.L4 && j < p.L)
              p.P[h * p.p_sh + int64_t(row0 + r) * p.p_sn + j] = __uint_as_float(v[e]);
          }
        }
      }
    }
    if (r == 0) bulk_wait<0>();
  } else if (warp == 8) {
    // ============================================= TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmKt);
      int khead[2] = {-1, -1};
      int issued = 0;
      for (int i = 0; i < n_local; ++i) {
        const int st = i % C::NSTAGE;
        const uint32_t ph = uint32_t((i / C::NSTAGE) & 1);
        if (!wait_bounded(BAR(2 + st), ph ^ 1u, ctl)) break;
        const int u = u0 + i, h = u / p.tiles, tile = u - h * p.tiles;
        const bool newk = khead[st] != h;
        const uint32_t sQ = sStage + uint32_t(st * C::STAGE_BYTES), sK = sQ + C::Q_BYTES;
        mbar_arrive_expect_tx(BAR(0 + st),
                              uint32_t(C::Q_BYTES + (newk ? C::NCH * p.Lpad * C::ROWB : 0)));
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          tma_load_4d(sQ + c * C::Q_CHUNK, &tmQ, BAR(0 + st), c * C::CH, tile * 128, h, p.b);
          if (newk) tma_load_4d(sK + c * C::K_CHUNK, &tmKt, BAR(0 + st), c * C::CH, 0, h, p.b);
        }
        khead[st] = h;
        issued = i + 1;
      }
      // every copy has landed before the CTA leaves (already true unless a
      // role aborted before consuming it)
      for (int i = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); i < issued; ++i)
        wait_drain(BAR(0 + i % C::NSTAGE), uint32_t((i / C::NSTAGE) & 1), kXDrainNs);
    }
  } else {
    // ============================================= MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, p.Lpad, 0, 0);
      constexpr uint32_t SBO = 8u * C::ROWB;
      bool ok = true;
      for (int i = 0; i < n_local && ok; ++i) {
        const int st = i % C::NSTAGE, buf = i & 1;
        if (!(ok = wait_bounded(BAR(0 + st), uint32_t((i / C::NSTAGE) & 1), ctl))) break;
        if (!(ok = wait_bounded(BAR(6 + buf), uint32_t(((i >> 1) & 1) ^ 1), ctl))) break;
        tc_fence_after();
        const uint32_t sQ = sStage + uint32_t(st * C::STAGE_BYTES), sK = sQ + C::Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int chunk = (kk * 16) / C::CH;
          const uint32_t within = uint32_t(((kk * 16) % C::CH) * 2);
          mma_ss(tmem + uint32_t(buf * 256),
                 smem_desc(sQ + chunk * C::Q_CHUNK + within, 16u, SBO, C::LAYOUT),
                 smem_desc(sK + chunk * C::K_CHUNK + within, 16u, SBO, C::LAYOUT), idesc,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(BAR(4 + buf));
        tc_commit(BAR(2 + st));
      }
      // every MMA has completed before TMEM is freed, whoever aborted
      tc_commit(BAR(8));
      wait_drain(BAR(8), 0u, kXDrainNs);
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
static safedit_status launch_x(const CUtensorMap& a, const CUtensorMap& k, const CUtensorMap& pm,
                               const XParams& p, cudaStream_t s) {
  auto kern = xattn_probs_kernel<D>;
  safedit_status st = set_smem(reinterpret_cast<const void*>(kern), XCfg<D>::SMEM_BYTES);
  if (st != SAFEDIT_OK) return st;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.units < sms ? p.units : sms;
  kern<<<grid, 320, XCfg<D>::SMEM_BYTES, s>>>(a, k, pm, p);
  return after_launch(1);
}

}  // namespace sd

using namespace sd;

extern "C" safedit_status safedit_cross_attn_probs(const safedit_tensor* q_img,
                                                   const safedit_tensor* k_txt,
                                                   const uint8_t* d_key_valid,
                                                   int32_t batch_index, float scale,
                                                   const safedit_tensor* p_out, void* stream) {
  safedit_status st;
  for (const safedit_tensor* t : {q_img, k_txt}) {
    if ((st = check_tensor(t, 4)) != SAFEDIT_OK) return st;
    if (t->dtype != SAFEDIT_BF16) return SAFEDIT_ERR_DTYPE;
    if (t->strides[3] != 1 || !aligned16(t->data)) return SAFEDIT_ERR_ALIGNMENT;
    for (int i = 0; i < 3; ++i)
      if (t->strides[i] % 8 != 0 || t->strides[i] < 0) return SAFEDIT_ERR_ALIGNMENT;
  }
  if ((st = check_tensor(p_out, 3)) != SAFEDIT_OK) return st;
  if (!d_key_valid) return SAFEDIT_ERR_INVALID_ARG;
  const int64_t B = q_img->dims[0], H = q_img->dims[1], N = q_img->dims[2], D = q_img->dims[3];
  const int64_t L = k_txt->dims[2];
  if (k_txt->dims[0] != B || k_txt->dims[1] != H || k_txt->dims[3] != D) return SAFEDIT_ERR_SHAPE;
  if (batch_index < 0 || batch_index >= B) return SAFEDIT_ERR_INVALID_ARG;
  if (D != 64 && D != 96 && D != 128) return SAFEDIT_ERR_UNSUPPORTED;
  if (L < 1 || L > 256) return SAFEDIT_ERR_UNSUPPORTED;
  if (p_out->dtype != SAFEDIT_F32) return SAFEDIT_ERR_DTYPE;
  if (p_out->dims[0] != H || p_out->dims[1] != N || p_out->dims[2] != L) return SAFEDIT_ERR_SHAPE;
  if (p_out->strides[2] != 1 || p_out->strides[1] % 4 != 0 || p_out->strides[0] % 4 != 0 ||
      !aligned16(p_out->data))
    return SAFEDIT_ERR_ALIGNMENT;
  if (N == 0 || H == 0) return SAFEDIT_OK;
  if (H > 65535) return SAFEDIT_ERR_SHAPE;
  XParams p{};
  p.key_valid = d_key_valid + int64_t(batch_index) * L;
  p.L = static_cast<int>(L);
  p.L4 = static_cast<int>(L & ~int64_t(3));
  p.P = static_cast<float*>(p_out->data);
  p.p_sh = p_out->strides[0];
  p.p_sn = p_out->strides[1];
  p.Lpad = static_cast<int>((L + 31) / 32 * 32);  // MMA N and TMEM chunks of 32 columns
  p.N = static_cast<int>(N);
  p.H = static_cast<int>(H);
  p.b = batch_index;
  p.tiles = static_cast<int>((N + 127) / 128);
  if (int64_t(p.tiles) * H > INT32_MAX) return SAFEDIT_ERR_SHAPE;
  p.units = p.tiles * p.H;
  const float sc = (scale > 0.f) ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale_log2 = sc * kXLog2e;
  p.wait_limit = wait_limit_ns();
  const int ch = (D % 64 == 0) ? 64 : 32;
  const CUtensorMapSwizzle swz = ch == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap tq, tk, tp{};
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
  if (p.L4 > 0) {
    const uint64_t dims[3] = {uint64_t(p.L4), uint64_t(N), uint64_t(H)};
    const uint64_t str[2] = {uint64_t(p_out->strides[1]) * 4, uint64_t(p_out->strides[0]) * 4};
    const uint32_t box[3] = {32u, 128u, 1u};
    if ((st = encode_tmap(&tp, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p_out->data, dims, str, box,
                          CU_TENSOR_MAP_SWIZZLE_128B)) != SAFEDIT_OK)
      return st;
  }
  p.status = status_ptr();
  if (!p.status) return SAFEDIT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (D) {
    case 64: return launch_x<64>(tq, tk, tp, p, s);
    case 96: return launch_x<96>(tq, tk, tp, p, s);
    default: return launch_x<128>(tq, tk, tp, p, s);
  }
}
