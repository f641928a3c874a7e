// attn.cu -- SRSU subset attention and CAR dense anchor on sm_100a.
//
// SAFE-DiT summary (gist.science 2606.29360), 방법론 3 / Italian page
// Metodologia 3: on a non-anchor step only the sensitive query rows are
// updated, and they attend over the global key/value set (fresh sensitive
// states plus cached context states); an anchor step refreshes every row.
// AccelAes summary (gist.science 2603.12575), B.2 SkipSparse: queries only on
// focus tokens, keys and values from the whole image.
//
//   o_r = sum_j softmax_j(scale q_{idx[r]} . k_j + pad_j + bias_{idx[r],j}) v_j
//
// Design (one CTA per SM, 384 threads = 3 warpgroups):
//   * 2 query tiles of 128 rows (256 rows per CTA).  The softmax warpgroup of
//     tile t (warps 4t..4t+3) gathers its rows q[idx[r]] with 16-byte
//     cp.async copies straight into the swizzled K-major shared-memory layout
//     the tensor core reads (the indexed gather replaces a copy of Q_S).
//   * the third warpgroup: warp 8 streams K and V tiles (128 keys) through an
//     NS-stage TMA ring, warp 9 issues tcgen05.mma, warps 10-11 only lend
//     their registers (setmaxnreg: 208 per softmax thread, 88 per control
//     thread).
//   * MMAs: S_t = Q_t K_j^T into TMEM (fp32, 128 columns per tile) and
//     O_t += P_t V_j with P_t read back from TMEM (the bf16 probabilities
//     overwrite S_t in place), so P never touches shared memory; issue order
//     per key tile PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), so one tile's
//     softmax overlaps the other tile's MMAs.  Descriptors are built once.
//   * softmax: thread = query row = TMEM lane.  Online softmax in base 2 with
//     a lazy rescale (the running max only moves when it grows by more than
//     2^8, which is exact after the final division by the row sum); packed
//     f32x2 FMAs and adds, three-input max; a quarter of the exponentials on
//     the FMA pipe (degree-3 polynomial), the rest on the MUFU unit.
//   * kept masks (template PAD / BIAS): logits scale s + pad + bias in one
//     packed FMA per pair; the pad one key tile ahead in a shared three-slot
//     ring, the bias one pass ahead through per-warp cp.async staging; each
//     key tile in passes of 64 (f32 bias: 32) columns; key tiles whose pad is
//     -inf throughout are skipped by every role; every exponential on MUFU.
//   * schedule: units of 256 query rows of one (b, h) slice.  A plain call
//     runs every unit whole; the tail-balanced call runs the units that fill
//     whole waves in one launch and cuts the last wave's units into key-range
//     parts (a second launch, SPLIT, overlapping the first one's drain by
//     programmatic dependent launch) whose partial O, max and sum
//     attn_merge_kernel combines.
// Every mbarrier wait is bounded; an expired wait raises the CTA's abort
// flag, drains in-flight TMA loads and MMAs, frees TMEM and returns.
#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace sd {

template <int D>
struct AttnCfg {
  static constexpr int BM = 128;                       // query rows per tile
  static constexpr int BN = 128;                       // keys per tile
  static constexpr int CH = (D % 64 == 0) ? 64 : 32;   // elements per swizzle chunk row
  static constexpr int NCH = D / CH;                   // chunks per row
  static constexpr int ROWB = CH * 2;                  // bytes per chunk row
  static constexpr uint32_t LAYOUT = (CH == 64) ? 2u : 4u;  // 128B / 64B swizzle
  static constexpr int CHUNK_BYTES = 128 * ROWB;       // one chunk of a 128-row tile
  static constexpr int TILE_BYTES = NCH * CHUNK_BYTES; // 128 rows x D bf16
  static constexpr int NS = (D == 64) ? 4 : (D == 96 ? 3 : 2);  // K/V ring depth
  static constexpr int UNITS = D * 2 / 16;             // 16-byte units per row
  static constexpr int SMEM_TILES = 2 + 2 * NS;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + SMEM_TILES * TILE_BYTES + BAR_BYTES;
  static constexpr int PAD_BYTES = 3 * 128 * 4 + 128;  // pad of 3 key tiles (all warps) + live-tile bits
  static constexpr int BIAS_BYTES = 8 * 32 * 128;      // per warp: 32 rows x 128 bytes
  static_assert(SMEM_BYTES + BIAS_BYTES + PAD_BYTES <= 232448, "shared memory");
  static_assert(D == 64 || D == 96 || D == 128, "head dim");
  static_assert(256 + 2 * D <= 512, "TMEM columns");
};

struct AttnParams {
  const __nv_bfloat16* q;
  int64_t q_sb, q_sh, q_sr;  // element strides
  const int* idx;            // nullable
  int n_rows, Nq, Nk, H;
  float scale;               // softmax scale
  float scale_log2;          // scale * log2(e)
  const float* pad;          // nullable, [B, Nk]
  int64_t pad_sb;
  const void* bias;          // nullable
  int bias_f32;
  int64_t bias_sb, bias_sh, bias_sq;
  __nv_bfloat16* out;
  int64_t o_sb, o_sh, o_sr;
  int out_scattered;
  int* status;
  uint64_t wait_limit;
  // Schedule: unit u = (row block u % n_rb, slice u / n_rb) of 256 query rows.
  // Units below n_full run whole (one launch, a whole number of waves when
  // split); every later unit runs as `split` CTAs of a second launch over
  // consecutive parts of the key tiles, which write their unnormalised O,
  // running max and row sum to `part` for attn_merge_kernel.
  int n_rb, n_full, split;
  float* part;  // [(unit - n_full) * split + part][256][D] O, then [..][256][2] (m, l)
  int n_part_units;
};

// 12 warps: two softmax warpgroups (warps 0-7), then TMA producer (8), MMA
// issuer (9) and two spare warps (10, 11) completing the third warpgroup, so
// that setmaxnreg can move registers from the control warpgroup (88 each) to
// the softmax warpgroups (208 each): 256*208 + 128*88 = 384*168.  The
// kept-mask kernels hold half a key tile of scores at a time and split
// 192 / 120 (256*192 + 128*120 = 384*168), which leaves them (nearly)
// spill-free.
constexpr int kAttnThreads = 384;
constexpr uint32_t kSoftmaxRegs = 208, kControlRegs = 88;
constexpr uint32_t kSoftmaxRegsMasked = 192, kControlRegsMasked = 120;
static_assert(256 * kSoftmaxRegs + 128 * kControlRegs <= 384 * 168, "register split");
static_assert(256 * kSoftmaxRegsMasked + 128 * kControlRegsMasked <= 384 * 168, "register split");
// Column pairs (bit e of the mask = pair e of each 16-pair group) whose
// exponentials go to the FMA-pipe polynomial instead of the MUFU unit, on the
// mask-free path.  Balances the two pipes (measured on B200 at the 2560^2
// SRSU launch: 1/4 of the pairs is best, 1/2 is slower than none).  Kept
// masks put every exponential on the MUFU unit (measured faster there: the
// mask terms already load the FMA pipe), which also gives masked keys their
// exact zero weight.
#ifndef SAFEDIT_EXP2_FMA_MASK
#define SAFEDIT_EXP2_FMA_MASK 0x8888u
#endif
constexpr uint32_t kExp2FmaMask = SAFEDIT_EXP2_FMA_MASK;
constexpr uint64_t kDrainNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Key tiles whose pad is -inf throughout carry exactly zero weight and are
// skipped (a bitmask of live tiles in shared memory; up to 1024 tiles).
constexpr int kLiveWords = 32;

__device__ __forceinline__ uint32_t swizzle_off(uint32_t off, uint32_t layout) {
  return layout == 2u ? (off ^ (((off >> 7) & 7u) << 4)) : (off ^ (((off >> 7) & 3u) << 4));
}

// Kept-bias element type (template parameter of the kernel).
constexpr int kBiasNone = 0, kBiasBf16 = 1, kBiasF32 = 2;

// Four pad values starting at key `k0` (a multiple of 4); zero past Nk.
__device__ __forceinline__ float4 load_pad4(const float* row, int k0, int Nk) {
  if (k0 + 4 <= Nk) return __ldg(reinterpret_cast<const float4*>(row + k0));
  float v[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] = (k0 + e < Nk) ? __ldg(row + k0 + e) : 0.f;
  return make_float4(v[0], v[1], v[2], v[3]);
}

// Asynchronous 16-byte global -> shared copy (no register staging); bytes
// past `src_bytes` are zero-filled and not read.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Stages the bias of this warp's 32 query rows, one 128-byte row segment
// each (64 bf16 or 32 f32 keys from key k0), into the warp's 4 KB buffer with
// coalesced copies (each instruction moves four row segments).  Row rr's
// 16-byte chunk ch lands in slot ch ^ (rr & 7) of the row's 128 bytes, so
// that the row-per-thread reads back are free of bank conflicts.  qrow[i] is
// the query index of row 4 i + lane / 8 (negative: no row); keys past Nk are
// zero-filled or skipped.
template <typename T>
__device__ __forceinline__ void stage_bias(uint32_t buf, const T* base, int64_t sq, const int (&qrow)[8],
                                           int k0, int Nk, int lane) {
  constexpr int EPC = 16 / int(sizeof(T));  // elements per 16-byte chunk
  const int ch = lane & 7;
  const int left = Nk - (k0 + ch * EPC);
  if (left > 0) {
    const uint32_t bytes = left >= EPC ? 16u : uint32_t(left) * uint32_t(sizeof(T));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int rr = 4 * i + (lane >> 3);
      if (qrow[i] >= 0)
        cp_async16(buf + uint32_t(rr * 128 + ((ch ^ (rr & 7)) << 4)),
                   base + int64_t(qrow[i]) * sq + k0 + ch * EPC, bytes);
    }
  }
  cp_async_commit();
}

template <int D, bool PAD, int BIAS, bool SPLIT>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_subset_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = AttnCfg<D>;
  constexpr bool MASKED = PAD || BIAS != kBiasNone;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase;                               // 2 tiles
  const uint32_t sK = sbase + 2 * C::TILE_BYTES;           // NS tiles
  const uint32_t sV = sK + C::NS * C::TILE_BYTES;          // NS tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_TILES * C::TILE_BYTES);
  const uint32_t b0 = smem_u32(bars);
  auto BAR = [&](int i) { return b0 + 8u * uint32_t(i); };
  const int Q_FULL = 0, K_FULL = 2, K_EMPTY = K_FULL + C::NS, V_FULL = K_EMPTY + C::NS,
            V_EMPTY = V_FULL + C::NS, S_FULL = V_EMPTY + C::NS, P_FULL = S_FULL + 2,
            O_FULL = P_FULL + 2, DRAIN = O_FULL + 1, NBARS = DRAIN + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // whole units: 2D grid (x: row block, y: slice), units from n_full on left
  // to the part launch; parts: CTA i runs part i % split of unit
  // n_full + i / split (recomputed where needed rather than kept live
  // through the main loop).  A whole-unit CTA lets a dependent launch (the
  // parts, which read only what it reads) start as soon as it is resident,
  // so the parts fill the SMs its last wave frees.
  if constexpr (!SPLIT) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (!SPLIT && int(blockIdx.y) * p.n_rb + int(blockIdx.x) >= p.n_full) return;
  auto decode = [&](int& unit_out, int& kpart_out) {
    if (SPLIT) {
      unit_out = p.n_full + int(blockIdx.x) / p.split;
      kpart_out = int(blockIdx.x) - (int(blockIdx.x) / p.split) * p.split;
    } else {
      unit_out = int(blockIdx.y) * p.n_rb + int(blockIdx.x);
      kpart_out = -1;
    }
  };
  int unit, kpart;
  decode(unit, kpart);
  const int bh = SPLIT ? unit / p.n_rb : int(blockIdx.y);
  const int b = bh / p.H, h = bh - b * p.H;
  const int row0 = SPLIT ? (unit - bh * p.n_rb) * 256 : int(blockIdx.x) * 256;
  const int nk = (p.Nk + C::BN - 1) / C::BN;
  // this CTA's key tiles [k_lo, k_hi)
  const int k_lo = !SPLIT || kpart < 0 ? 0 : int(int64_t(nk) * kpart / p.split);
  const int k_hi = !SPLIT || kpart < 0 ? nk : int(int64_t(nk) * (kpart + 1) / p.split);
  // live key tiles (kept key padding): a tile whose pad entries are all -inf
  // adds nothing to any row (its weights are exactly zero) and is skipped by
  // every role; every role walks the same bitmask, so they agree on the
  // sequence of tiles
  uint32_t* const live_bits = reinterpret_cast<uint32_t*>(
      smem + C::SMEM_TILES * C::TILE_BYTES + C::BAR_BYTES + (BIAS != kBiasNone ? C::BIAS_BYTES : 0) +
      3 * 128 * 4);
  const bool skip_tiles = PAD && nk <= kLiveWords * 32;
  if constexpr (PAD) {
    if (threadIdx.x < kLiveWords) live_bits[threadIdx.x] = 0u;
    __syncthreads();
    if (skip_tiles) {
      const float* pr = p.pad + b * p.pad_sb;
      for (int j = threadIdx.x >> 5; j < nk; j += kAttnThreads / 32) {
        bool live = false;
        for (int c = lane; c < C::BN && j * C::BN + c < p.Nk; c += 32)
          live |= !(__ldg(pr + j * C::BN + c) == -INFINITY);
        if (__any_sync(0xffffffffu, live) && lane == 0) atomicOr(live_bits + (j >> 5), 1u << (j & 31));
      }
    }
  }
  const uint32_t live_s = smem_u32(live_bits);
  auto live_word = [&](int w) -> uint32_t {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(live_s + uint32_t(w) * 4u));
    return v;
  };
  // first live tile at or after j (nk if none)
  auto next_live = [&](int j) -> int {
    if (!skip_tiles) return j;
    while (j < nk) {
      const uint32_t w = live_word(j >> 5) >> (j & 31);
      if (w) return j + __ffs(w) - 1;
      j = (j | 31) + 1;
    }
    return nk;
  };
  // live tiles in [k_lo, k_hi)
  auto live_count = [&]() -> int {
    if (!skip_tiles) return k_hi - k_lo;
    int n = 0;
    for (int w = k_lo >> 5; w <= (k_hi - 1) >> 5; ++w) {
      uint32_t bits = live_word(w);
      if (w == (k_lo >> 5)) bits &= ~0u << (k_lo & 31);
      if (w == ((k_hi - 1) >> 5) && (k_hi & 31)) bits &= ~(~0u << (k_hi & 31));
      n += __popc(bits);
    }
    return n;
  };

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(Q_FULL + t), 128);
      mbar_init(BAR(S_FULL + t), 1);
      mbar_init(BAR(P_FULL + t), 128);
    }
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(K_FULL + s), 1);
      mbar_init(BAR(K_EMPTY + s), 1);
      mbar_init(BAR(V_FULL + s), 1);
      mbar_init(BAR(V_EMPTY + s), 1);
    }
    mbar_init(BAR(O_FULL), 1);
    mbar_init(BAR(DRAIN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 9 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit};

  if (warp < 8) {
    // ================================================== softmax warpgroups
    setmaxnreg_inc<MASKED ? kSoftmaxRegsMasked : kSoftmaxRegs>();
    const int t = warp >> 2;            // query tile
    const int wr = warp & 3;            // TMEM lane quarter
    const int tid = threadIdx.x & 127;  // thread within the warpgroup
    const int tile_row0 = row0 + t * 128;
    // ---- indexed gather of the tile's query rows: 16-byte cp.async copies
    // (no register staging) straight into the swizzled K-major layout
    {
      const uint32_t qs = sQ + t * C::TILE_BYTES;
      const __nv_bfloat16* qbh = p.q + b * p.q_sb + h * p.q_sh;
      constexpr int UPC = C::ROWB / 16;  // units per chunk row
      for (int u = tid; u < 128 * C::UNITS; u += 128) {
        const int rr = u / C::UNITS, cu = u - rr * C::UNITS;
        const int gr = tile_row0 + rr;
        const __nv_bfloat16* src = qbh;  // not read when nothing is copied (zero fill)
        uint32_t bytes = 0u;
        if (gr < p.n_rows) {
          const int qi = p.idx ? __ldg(p.idx + gr) : gr;
          if (qi >= 0 && qi < p.Nq) {
            src = qbh + int64_t(qi) * p.q_sr + cu * 8;
            bytes = 16u;
          } else if (cu == 0) {
            set_status(p.status, SAFEDIT_ERR_INDEX);
          }
        }
        const int chunk = cu / UPC, cin = cu - chunk * UPC;
        const uint32_t off = uint32_t(chunk * C::CHUNK_BYTES) +
                             swizzle_off(uint32_t(rr * C::ROWB + cin * 16), C::LAYOUT);
        cp_async16(qs + off, src, bytes);
      }
      cp_async_commit();
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(BAR(Q_FULL + t));
    }

    const uint32_t lane_base = uint32_t(wr * 32) << 16;
    const uint32_t tS = tmem + uint32_t(t * 128) + lane_base;
    const uint32_t tO = tmem + 256u + uint32_t(t * D) + lane_base;
    const int my_row = tile_row0 + wr * 32 + lane;
    int my_q = -1;  // query index of this thread's row, -1 if none
    if (my_row < p.n_rows) {
      my_q = p.idx ? __ldg(p.idx + my_row) : my_row;
      if (my_q < 0 || my_q >= p.Nq) my_q = -1;
    }
    const float sl2 = p.scale_log2;
    // Kept masks.  Their operands for the next key columns are fetched ahead,
    // so that the load latency overlaps the current columns instead of
    // sitting between S and P.  The pad: one tile ahead, one 16-byte load per
    // lane into a three-slot ring (slot = tile mod 3, 1.5 KB) shared by all
    // eight softmax warps, read back as broadcasts.  Every warp writes the
    // same values there (before waiting for the tile's S) and reads them after
    // its own __syncwarp.  A warp that writes tile j + 1 has finished tile j,
    // whose S needed P(j - 1) of its own query tile and P(j - 2) of the other
    // (the MMA issue order), so every other warp is reading tile j - 1 or
    // later: slots j - 1, j and j + 1 are distinct.
    // A bias: one pass (64 bf16 or 32 f32 keys) ahead, copied asynchronously
    // and coalesced into this warp's 4 KB buffer, read back row per thread.
    uint8_t* const mask_smem = smem + C::SMEM_TILES * C::TILE_BYTES + C::BAR_BYTES;
    const uint32_t bias_buf = smem_u32(mask_smem) + uint32_t(warp * 4096);
    const uint32_t pad_buf = smem_u32(mask_smem) + uint32_t(BIAS != kBiasNone ? C::BIAS_BYTES : 0);
    const float* const pad_row = PAD ? p.pad + b * p.pad_sb : nullptr;
    float4 pad_next = make_float4(0.f, 0.f, 0.f, 0.f);
    const int n_live = live_count();
    int j_first = next_live(k_lo);
    if constexpr (PAD) pad_next = load_pad4(pad_row, j_first * C::BN + 4 * lane, p.Nk);
    using BiasT = typename std::conditional<BIAS == kBiasF32, float, __nv_bfloat16>::type;
    const BiasT* const bias_bh =
        BIAS != kBiasNone
            ? static_cast<const BiasT*>(p.bias) + b * p.bias_sb + h * p.bias_sh
            : nullptr;
    int qrow[8];  // query index of row 4 i + lane / 8 of this warp (bias staging)
    if constexpr (BIAS != kBiasNone) {
#pragma unroll
      for (int i = 0; i < 8; ++i) qrow[i] = __shfl_sync(0xffffffffu, my_q, 4 * i + (lane >> 3));
      stage_bias(bias_buf, bias_bh, p.bias_sq, qrow, j_first * C::BN, p.Nk, lane);
    }
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int pad_slot = 0;  // it mod 3
    // it counts the live key tiles processed (it drives the barrier phases),
    // j is the key tile itself
    int j = j_first;
    for (int it = 0; it < n_live; ++it) {
      const int key0 = j * C::BN;
      const int j_next = next_live(j + 1);
      if constexpr (PAD) {
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                         pad_buf + uint32_t(pad_slot * 512 + lane * 16)),
                     "f"(pad_next.x), "f"(pad_next.y), "f"(pad_next.z), "f"(pad_next.w)
                     : "memory");
        __syncwarp();
        if (j_next < nk) pad_next = load_pad4(pad_row, j_next * C::BN + 4 * lane, p.Nk);
      }
      if (!wait_warp(BAR(S_FULL + t), uint32_t(it & 1), ctl)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // The mask-free path takes the tile's 128 columns in one pass.  With
      // kept masks the tile goes in passes of 64 columns (32 with an f32
      // bias: one 128-byte bias row segment per pass), each with its own
      // online-softmax max, which keeps the mask operands of a pass in
      // registers beside its scores; when a pass raises the running max, the
      // earlier passes' P (already in TMEM) is rescaled with it.
      constexpr int NH = !MASKED ? 1 : (BIAS == kBiasF32 ? 4 : 2), HW = 128 / NH;
      // one pass over columns [hf * HW, hf * HW + HW); hf is a compile-time
      // constant, so every register array below is indexed statically
      auto pass = [&](auto hf_tag) {
        constexpr int hf = decltype(hf_tag)::value;
        constexpr int c0 = hf * HW;  // first column of the pass
        // x = raw scores (mask-free) or natural-unit logits
        // scale * s + pad + bias (kept masks)
        float x[HW];
        {
          uint32_t r[HW / 32][32];
#pragma unroll
          for (int q4 = 0; q4 < HW / 32; ++q4) tmem_ld32(tS + uint32_t(c0 + q4 * 32), r[q4]);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < HW / 32; ++q4)
#pragma unroll
            for (int e = 0; e < 32; ++e) x[q4 * 32 + e] = __uint_as_float(r[q4][e]);
        }
        if constexpr (MASKED) {
          const uint64_t sc2 = f2_pack(p.scale, p.scale);
          const int lim = p.Nk - key0 - c0;
          if constexpr (BIAS != kBiasNone) {  // this pass's bias has landed
            cp_async_wait_all();
            __syncwarp();
          }
#pragma unroll
          for (int c = 0; c < HW; c += 8) {
            float add[8];
            if constexpr (PAD) {
              const uint32_t ps = pad_buf + uint32_t(pad_slot * 512 + (c0 + c) * 4);
              asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                           : "=f"(add[0]), "=f"(add[1]), "=f"(add[2]), "=f"(add[3])
                           : "r"(ps));
              asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                           : "=f"(add[4]), "=f"(add[5]), "=f"(add[6]), "=f"(add[7])
                           : "r"(ps + 16u));
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) add[e] = 0.f;
            }
            if constexpr (BIAS == kBiasBf16) {
              uint32_t ws[4];
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(ws[0]), "=r"(ws[1]), "=r"(ws[2]), "=r"(ws[3])
                           : "r"(bias_buf + uint32_t(lane * 128 + (((c / 8) ^ (lane & 7)) << 4))));
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                add[2 * e] += __uint_as_float(ws[e] << 16);
                add[2 * e + 1] += __uint_as_float(ws[e] & 0xFFFF0000u);
              }
            } else if constexpr (BIAS == kBiasF32) {
#pragma unroll
              for (int hc = 0; hc < 2; ++hc) {
                float w[4];
                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(w[0]), "=f"(w[1]), "=f"(w[2]), "=f"(w[3])
                             : "r"(bias_buf +
                                   uint32_t(lane * 128 + (((c / 4 + hc) ^ (lane & 7)) << 4))));
#pragma unroll
                for (int e = 0; e < 4; ++e) add[4 * hc + e] += w[e];
              }
            }
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float y0, y1;
              f2_unpack(f2_fma(f2_pack(x[c + e], x[c + e + 1]), sc2, f2_pack(add[e], add[e + 1])),
                        y0, y1);
              x[c + e] = y0;
              x[c + e + 1] = y1;
            }
          }
          if constexpr (BIAS != kBiasNone) {
            // every lane has read the buffer: stage the next pass into it
            __syncwarp();
            const int k_next = (hf + 1 < NH) ? key0 + c0 + HW : j_next * C::BN;
            if (k_next < nk * C::BN) stage_bias(bias_buf, bias_bh, p.bias_sq, qrow, k_next, p.Nk, lane);
          }
        }
        if (key0 + C::BN > p.Nk) {  // ragged last key tile
          const int lim = p.Nk - key0 - c0;
#pragma unroll
          for (int c = 0; c < HW; ++c)
            if (c >= lim) x[c] = -INFINITY;
        }
        // row max of the pass (in log2 units)
        float mt;
        {
          // four independent max chains (latency), three-input max (issue)
          float m0 = fmaxf(x[0], x[1]), m1 = fmaxf(x[2], x[3]), m2 = fmaxf(x[4], x[5]),
                m3 = fmaxf(x[6], x[7]);
#pragma unroll
          for (int c = 8; c < HW; c += 8) {
            m0 = max3(m0, x[c], x[c + 1]);
            m1 = max3(m1, x[c + 2], x[c + 3]);
            m2 = max3(m2, x[c + 4], x[c + 5]);
            m3 = max3(m3, x[c + 6], x[c + 7]);
          }
          mt = fmaxf(max3(m0, m1, m2), m3);
          // the max commutes with the positive factor into log2 units
          mt *= MASKED ? kLog2e : sl2;
        }
        // lazy rescale: the running max moves only when it grows by > 2^8
        bool need_o = false, raised = false;
        float alpha = 1.f;
        if (mt > m_run + kRescaleThreshold) {
          alpha = ex2_approx(m_run - mt);  // 0 when m_run = -inf
          l_run *= alpha;
          m_run = mt;
          need_o = (it > 0);
          raised = true;
        }
        if (__any_sync(0xffffffffu, need_o)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + uint32_t(c * 32), r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(tO + uint32_t(c * 32), r);
          }
        }
        if constexpr (hf > 0) {
          // the earlier passes' probabilities (hf * HW / 2 packed columns)
          constexpr int PCOLS = hf * HW / 2;
          if (__any_sync(0xffffffffu, raised)) {
            tmem_wait_st();
            if constexpr (PCOLS % 32 == 0) {
#pragma unroll
              for (int q = 0; q < PCOLS / 32; ++q) {
                uint32_t r[32];
                tmem_ld32(tS + uint32_t(q * 32), r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                  r[e] = pack_bf16x2(__uint_as_float(r[e] << 16) * alpha,
                                     __uint_as_float(r[e] & 0xFFFF0000u) * alpha);
                tmem_st32(tS + uint32_t(q * 32), r);
              }
            } else {
#pragma unroll
              for (int q = 0; q < PCOLS / 16; ++q) {
                uint32_t r[16];
                tmem_ld16(tS + uint32_t(q * 16), r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                  r[e] = pack_bf16x2(__uint_as_float(r[e] << 16) * alpha,
                                     __uint_as_float(r[e] & 0xFFFF0000u) * alpha);
                tmem_st16(tS + uint32_t(q * 16), r);
              }
            }
          }
        }
        const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
        const float mul = MASKED ? kLog2e : sl2;
        const uint64_t mul2 = f2_pack(mul, mul), negm2 = f2_pack(neg_m, neg_m);
        // four independent partial sums: the row sum is not one serial chain
        uint64_t sum2[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f),
                            f2_pack(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < HW / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t a2 =
                f2_fma(f2_pack(x[c * 32 + 2 * e], x[c * 32 + 2 * e + 1]), mul2, negm2);
            float a0, a1, p0, p1;
            f2_unpack(a2, a0, a1);
            if (!MASKED && ((kExp2FmaMask >> e) & 1u)) {
              exp2_pair_fma(a0, a1, p0, p1);
            } else {
              p0 = ex2_approx(a0);
              p1 = ex2_approx(a1);
            }
            sum2[e & 3] = f2_add(sum2[e & 3], f2_pack(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + uint32_t((c0 / 32 + c) * 16), pk);
        }
        {
          float s0, s1;
          f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), s0, s1);
          l_run += s0 + s1;
        }
      };
      pass(std::integral_constant<int, 0>{});
      if constexpr (NH > 1) pass(std::integral_constant<int, 1>{});
      if constexpr (NH > 2) {
        pass(std::integral_constant<int, 2>{});
        pass(std::integral_constant<int, 3>{});
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(P_FULL + t));
      j = j_next;
      pad_slot = (pad_slot == 2) ? 0 : pad_slot + 1;
    }
    if constexpr (BIAS != kBiasNone) cp_async_wait_all();  // none in flight at exit
    // ---- epilogue: O / l -> bf16 rows; for a key-range part of a split
    // unit, the unnormalised O, running max and row sum for the merge
    if (ok && wait_warp(BAR(O_FULL), 0u, ctl)) {
      tc_fence_after();
      int e_unit, e_part;
      decode(e_unit, e_part);
      const bool partial = SPLIT && e_part >= 0;
      const bool live = my_q >= 0;
      if (live && !partial && !(l_run > 0.f)) set_status(p.status, SAFEDIT_ERR_MASKED_ROW);
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      // with skipped key tiles O may never have been written: a row with no
      // weight (fully masked: an error, reported above; for a part, a key
      // range with no admissible key, left to the merge) is written as zeros
      const bool zero_row = PAD && !(l_run > 0.f);
      const int64_t slot = int64_t(e_unit - p.n_full) * p.split + e_part;
      const int rr = t * 128 + wr * 32 + lane;
      __nv_bfloat16* orow = nullptr;
      float* po = nullptr;
      if (live && partial) {
        po = p.part + (slot * 256 + rr) * D;
      } else if (live) {
        const int64_t orow_idx = p.out_scattered ? int64_t(my_q) : int64_t(my_row);
        orow = p.out + b * p.o_sb + h * p.o_sh + orow_idx * p.o_sr;
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + uint32_t(c * 32), r);
        tmem_wait_ld();
        if (live && partial) {
          float4* dst = reinterpret_cast<float4*>(po + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = zero_row ? make_float4(0.f, 0.f, 0.f, 0.f)
                              : make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                            __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
        } else if (live) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = zero_row ? 0u
                            : pack_bf16x2(__uint_as_float(r[2 * e]) * inv,
                                          __uint_as_float(r[2 * e + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      if (live && partial) {
        float* const pml = p.part + int64_t(p.n_part_units) * p.split * 256 * D + (slot * 256 + rr) * 2;
        pml[0] = m_run;
        pml[1] = l_run;
      }
    }
  } else {
    setmaxnreg_dec<MASKED ? kControlRegsMasked : kControlRegs>();
    if (warp == 8) {
      // ================================================ TMA producer (K, V)
      if (lane == 0) {
        int issued_k = 0, issued_v = 0;
        const int n_live = live_count();
        for (int it = 0, kt = next_live(k_lo); it < n_live; ++it, kt = next_live(kt + 1)) {
          const int s = it % C::NS;
          const uint32_t ph = uint32_t((it / C::NS) & 1);
          if (!wait_bounded(BAR(K_EMPTY + s), ph ^ 1u, ctl)) break;
          mbar_arrive_expect_tx(BAR(K_FULL + s), C::TILE_BYTES);
#pragma unroll
          for (int c = 0; c < C::NCH; ++c)
            tma_load_4d(sK + s * C::TILE_BYTES + c * C::CHUNK_BYTES, &tmK, BAR(K_FULL + s),
                        c * C::CH, kt * C::BN, h, b);
          issued_k = it + 1;
          if (!wait_bounded(BAR(V_EMPTY + s), ph ^ 1u, ctl)) break;
          mbar_arrive_expect_tx(BAR(V_FULL + s), C::TILE_BYTES);
#pragma unroll
          for (int c = 0; c < C::NCH; ++c)
            tma_load_4d(sV + s * C::TILE_BYTES + c * C::CHUNK_BYTES, &tmV, BAR(V_FULL + s),
                        c * C::CH, kt * C::BN, h, b);
          issued_v = it + 1;
        }
        // every copy has landed before the CTA leaves (already true unless a
        // role aborted before consuming it)
        for (int j = (issued_k > C::NS ? issued_k - C::NS : 0); j < issued_k; ++j)
          wait_drain(BAR(K_FULL + j % C::NS), uint32_t((j / C::NS) & 1), kDrainNs);
        for (int j = (issued_v > C::NS ? issued_v - C::NS : 0); j < issued_v; ++j)
          wait_drain(BAR(V_FULL + j % C::NS), uint32_t((j / C::NS) & 1), kDrainNs);
      }
    } else if (warp == 9) {
      // ================================================ MMA issuer
      if (lane == 0) {
        const uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
        const uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
        const uint32_t tS0 = tmem, tS1 = tmem + 128u;
        const uint32_t tO0 = tmem + 256u, tO1 = tmem + 256u + uint32_t(D);
        constexpr uint32_t SBO = 8u * C::ROWB;
        // Descriptors are built once; per MMA only the 16-byte address field
        // of the low word advances (all smem offsets here stay below 256 KB,
        // so the field never carries into the other fields).
        const uint64_t qd0 = smem_desc(sQ, 16u, SBO, C::LAYOUT);
        const uint64_t qd1 = smem_desc(sQ + C::TILE_BYTES, 16u, SBO, C::LAYOUT);
        const uint64_t kd0 = smem_desc(sK, 16u, SBO, C::LAYOUT);
        const uint64_t vd0 = smem_desc(sV, uint32_t(C::CHUNK_BYTES), SBO, C::LAYOUT);
        auto adv = [](uint64_t d, uint32_t bytes) {
          return (d & 0xFFFFFFFF00000000ull) | uint64_t(uint32_t(d) + (bytes >> 4));
        };
        auto issue_qk = [&](uint32_t d_tmem, uint64_t qd, uint64_t kd) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = uint32_t(((kk * 16) / C::CH) * C::CHUNK_BYTES + ((kk * 16) % C::CH) * 2);
            mma_ss(d_tmem, adv(qd, off), adv(kd, off), idesc_qk, kk > 0 ? 1u : 0u);
          }
        };
        auto issue_pv = [&](uint32_t d_tmem, uint32_t p_tmem, uint64_t vd, bool acc) {
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk)
            mma_ts(d_tmem, p_tmem + uint32_t(kk * 8), adv(vd, uint32_t(kk * 16 * C::ROWB)), idesc_pv,
                   (acc || kk > 0) ? 1u : 0u);
        };
        // n_live counts key tiles in issue order (all of them unless tiles of
        // -inf padding are skipped); no live tile: no MMA, O_FULL at once
        const int n_live = live_count();
        bool ok = wait_bounded(BAR(Q_FULL + 0), 0u, ctl) && wait_bounded(BAR(Q_FULL + 1), 0u, ctl) &&
                  (n_live == 0 || wait_bounded(BAR(K_FULL + 0), 0u, ctl));
        if (ok && n_live > 0) {
          tc_fence_after();
          issue_qk(tS0, qd0, kd0);
          tc_commit(BAR(S_FULL + 0));
          issue_qk(tS1, qd1, kd0);
          tc_commit(BAR(S_FULL + 1));
          tc_commit(BAR(K_EMPTY + 0));
        }
        for (int j = 0; ok && j < n_live; ++j) {
          const int s = j % C::NS;
          const uint32_t ph = uint32_t((j / C::NS) & 1);
          const bool more = (j + 1 < n_live);
          const int s1 = (j + 1) % C::NS;
          const uint32_t ph1 = uint32_t(((j + 1) / C::NS) & 1);
          if (!(ok = wait_bounded(BAR(V_FULL + s), ph, ctl))) break;
          if (!(ok = wait_bounded(BAR(P_FULL + 0), uint32_t(j & 1), ctl))) break;
          tc_fence_after();
          issue_pv(tO0, tS0, adv(vd0, uint32_t(s * C::TILE_BYTES)), j > 0);
          if (more) {
            if (!(ok = wait_bounded(BAR(K_FULL + s1), ph1, ctl))) break;
            tc_fence_after();
            issue_qk(tS0, qd0, adv(kd0, uint32_t(s1 * C::TILE_BYTES)));
            tc_commit(BAR(S_FULL + 0));
          }
          if (!(ok = wait_bounded(BAR(P_FULL + 1), uint32_t(j & 1), ctl))) break;
          tc_fence_after();
          issue_pv(tO1, tS1, adv(vd0, uint32_t(s * C::TILE_BYTES)), j > 0);
          tc_commit(BAR(V_EMPTY + s));
          if (more) {
            issue_qk(tS1, qd1, adv(kd0, uint32_t(s1 * C::TILE_BYTES)));
            tc_commit(BAR(S_FULL + 1));
            tc_commit(BAR(K_EMPTY + s1));
          }
        }
        if (ok) tc_commit(BAR(O_FULL));
        // every MMA has completed before TMEM is freed, whoever aborted
        tc_commit(BAR(DRAIN));
        wait_drain(BAR(DRAIN), 0u, kDrainNs);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // the part launch may overlap the whole-unit launch before it: its last CTA
  // leaves only once that launch has completed, so whatever follows in the
  // stream (the merge, then the caller's work) runs after both
  if constexpr (SPLIT) {
    if (threadIdx.x == 0 && blockIdx.x == gridDim.x - 1) asm volatile("griddepcontrol.wait;" ::: "memory");
  }
}

// Combines the key-range parts of the split units: per query row,
// m = max m_i, l = sum 2^(m_i - m) l_i, o = sum 2^(m_i - m) O_i / l (the same
// online-softmax merge the kernel applies between key tiles), written as a
// bf16 row where the whole unit would have written it.  One warp per row.
template <int D>
__global__ void __launch_bounds__(256) attn_merge_kernel(const AttnParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= int64_t(p.n_part_units) * 256) return;
  const int pu = int(row >> 8), rr = int(row & 255);
  const int unit = p.n_full + pu;
  const int bh = unit / p.n_rb;
  const int b = bh / p.H, h = bh - b * p.H;
  const int my_row = (unit - bh * p.n_rb) * 256 + rr;
  if (my_row >= p.n_rows) return;
  const int my_q = p.idx ? __ldg(p.idx + my_row) : my_row;
  if (my_q < 0 || my_q >= p.Nq) return;  // reported by the attention kernel
  const float* ml = p.part + int64_t(p.n_part_units) * p.split * 256 * D;
  float m = -INFINITY;
  for (int k = 0; k < p.split; ++k) m = fmaxf(m, ml[((int64_t(pu) * p.split + k) * 256 + rr) * 2]);
  const int64_t orow_idx = p.out_scattered ? int64_t(my_q) : int64_t(my_row);
  __nv_bfloat16* orow = p.out + b * p.o_sb + h * p.o_sh + orow_idx * p.o_sr;
  if (m == -INFINITY) {  // no part has an admissible key: a fully masked row
    if (lane == 0) set_status(p.status, SAFEDIT_ERR_MASKED_ROW);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) orow[lane + 32 * e] = __float2bfloat16_rn(0.f);
    return;
  }
  float l = 0.f, acc[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
  for (int k = 0; k < p.split; ++k) {
    const int64_t slot = int64_t(pu) * p.split + k;
    const float w = exp2f(ml[(slot * 256 + rr) * 2] - m);
    l = fmaf(w, ml[(slot * 256 + rr) * 2 + 1], l);
    const float* po = p.part + (slot * 256 + rr) * D;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) acc[e] = fmaf(w, po[lane + 32 * e], acc[e]);
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) orow[lane + 32 * e] = __float2bfloat16_rn(acc[e] * inv);
}

// Launch plan: units of 256 query rows, longest first.  When the units do
// not fill the last wave of the SMs, those last units are each split into
// s = 2..4 parts over the key tiles, run after the whole units (which then
// fill a whole number of waves).  A CTA costs about kFixedUs (set-up, TMEM,
// epilogue) plus kTileUs per key tile of 128 at d = 96 (measured on B200,
// one full wave, 1280..25600 keys; scaled by d / 96 for other widths).  The
// tail's ceil(tail s / SMs) rounds of 1/s units plus the merge must save 3%
// of the whole launch (its rounds of whole units) for a split to be taken:
// smaller predicted savings did not show on B200, where a power-capped
// launch runs its other SMs faster while the last round leaves some idle.
struct AttnPlan {
  int n_rb = 0, n_units = 0, n_full = 0, split = 1, n_part_units = 0;
  size_t ws_bytes = 0;
};

static int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    sms = 148;
  return sms;
}

static AttnPlan plan_attn(int64_t n_rows, int64_t BH, int64_t Nk, int D, bool splittable, int sms) {
  AttnPlan pl;
  pl.n_rb = int((n_rows + 255) / 256);
  pl.n_units = int(pl.n_rb * BH);
  pl.n_full = pl.n_units;
  const int64_t nk = (Nk + 127) / 128;
  const int tail = pl.n_units % sms;
  if (!splittable || tail == 0 || nk < 8) return pl;
  constexpr double kFixedUs = 11.6, kTileUs = 1.83, kMergeUs = 8.0;
  const double tile_us = kTileUs * D / 96.0;
  const double unit_us = kFixedUs + double(nk) * tile_us;
  const double rounds_whole = double((pl.n_units + sms - 1) / sms);
  double best = unit_us - 0.03 * rounds_whole * unit_us;
  for (int s = 2; s <= 4; ++s) {
    const double rounds = double((int64_t(tail) * s + sms - 1) / sms);
    const double cost = rounds * (kFixedUs + double(nk) * tile_us / s) + kMergeUs;
    if (cost < best) {
      best = cost;
      pl.split = s;
    }
  }
  if (pl.split == 1) return pl;
  pl.n_part_units = tail;
  pl.n_full = pl.n_units - tail;
  pl.ws_bytes = size_t(tail) * size_t(pl.split) * 256u * size_t(D + 2) * sizeof(float);
  return pl;
}

template <int D, bool PAD, int BIAS, bool SPLIT = false>
static safedit_status launch_attn(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                  const AttnParams& p, int B, cudaStream_t stream) {
  using C = AttnCfg<D>;
  auto kern = attn_subset_kernel<D, PAD, BIAS, SPLIT>;
  constexpr int smem_bytes =
      C::SMEM_BYTES + (BIAS != kBiasNone ? C::BIAS_BYTES : 0) + (PAD ? C::PAD_BYTES : 0);
  safedit_status st = set_smem(reinterpret_cast<const void*>(kern), smem_bytes);
  if (st != SAFEDIT_OK) return st;
  if (SPLIT) {
    // programmatic serialization after the whole-unit launch (when there is
    // one): the parts may start while its last wave drains
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(p.n_part_units * p.split));
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.n_full > 0 ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, tmK, tmV, p) != cudaSuccess) return SAFEDIT_ERR_CUDA;
  } else {
    (void)B;
    dim3 grid(p.n_rb, (p.n_full + p.n_rb - 1) / p.n_rb);
    kern<<<grid, kAttnThreads, smem_bytes, stream>>>(tmK, tmV, p);
  }
  return after_launch(1);
}

// A split plan: the whole units (a whole number of waves), then the parts of
// the last units, then their merge, in stream order.
template <int D, bool PAD, int BIAS>
static safedit_status launch_attn_split(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                        const AttnParams& p, int B, cudaStream_t stream) {
  safedit_status st = SAFEDIT_OK;
  if (p.n_full > 0 && (st = launch_attn<D, PAD, BIAS>(tmK, tmV, p, B, stream)) != SAFEDIT_OK) return st;
  if ((st = launch_attn<D, PAD, BIAS, true>(tmK, tmV, p, B, stream)) != SAFEDIT_OK) return st;
  attn_merge_kernel<D><<<(p.n_part_units * 256 + 7) / 8, 256, 0, stream>>>(p);
  return after_launch(1);
}

template <int D, bool PAD, int BIAS>
static safedit_status launch_planned(const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnParams& p,
                                     int B, cudaStream_t s) {
  if (p.n_part_units > 0) return launch_attn_split<D, PAD, BIAS>(tmK, tmV, p, B, s);
  return launch_attn<D, PAD, BIAS>(tmK, tmV, p, B, s);
}

template <int D>
static safedit_status dispatch_attn(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                    const AttnParams& p, int B, cudaStream_t s) {
  const bool pad = p.pad != nullptr;
  const int bias = p.bias == nullptr ? kBiasNone : (p.bias_f32 ? kBiasF32 : kBiasBf16);
  if (pad) {
    if (bias == kBiasBf16) return launch_planned<D, true, kBiasBf16>(tmK, tmV, p, B, s);
    if (bias == kBiasF32) return launch_planned<D, true, kBiasF32>(tmK, tmV, p, B, s);
    return launch_planned<D, true, kBiasNone>(tmK, tmV, p, B, s);
  }
  if (bias == kBiasBf16) return launch_planned<D, false, kBiasBf16>(tmK, tmV, p, B, s);
  if (bias == kBiasF32) return launch_planned<D, false, kBiasF32>(tmK, tmV, p, B, s);
  return launch_planned<D, false, kBiasNone>(tmK, tmV, p, B, s);
}

static safedit_status check_bhnd(const safedit_tensor* t) {
  safedit_status st = check_tensor(t, 4);
  if (st != SAFEDIT_OK) return st;
  if (t->dtype != SAFEDIT_BF16) return SAFEDIT_ERR_DTYPE;
  if (t->strides[3] != 1) return SAFEDIT_ERR_ALIGNMENT;
  for (int i = 0; i < 3; ++i)
    if (t->strides[i] % 8 != 0 || t->strides[i] < 0) return SAFEDIT_ERR_ALIGNMENT;
  if (!aligned16(t->data)) return SAFEDIT_ERR_ALIGNMENT;
  return SAFEDIT_OK;
}

static safedit_status make_kv_map(CUtensorMap* m, const safedit_tensor* t, int D) {
  const int ch = (D % 64 == 0) ? 64 : 32;
  const uint64_t dims[4] = {uint64_t(t->dims[3]), uint64_t(t->dims[2]), uint64_t(t->dims[1]),
                            uint64_t(t->dims[0])};
  const uint64_t strides[3] = {uint64_t(t->strides[2]) * 2, uint64_t(t->strides[1]) * 2,
                               uint64_t(t->strides[0]) * 2};
  const uint32_t box[4] = {uint32_t(ch), 128u, 1u, 1u};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box,
                     ch == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

}  // namespace sd

using namespace sd;

// Shared body of safedit_attn_subset (ws == NULL: whole units only) and
// safedit_attn_subset_ws (the tail of the launch split over the keys when
// the plan asks for it and the workspace holds the partial results).
static safedit_status attn_subset_impl(const safedit_tensor* q, const safedit_tensor* k,
                                       const safedit_tensor* v, const int32_t* d_idx, int32_t n_idx,
                                       const safedit_tensor* key_pad, const safedit_tensor* bias,
                                       float scale, const safedit_tensor* out, int32_t out_scattered,
                                       void* d_ws, size_t ws_bytes, bool use_ws, void* stream) {
  safedit_status st;
  if ((st = check_bhnd(q)) != SAFEDIT_OK) return st;
  if ((st = check_bhnd(k)) != SAFEDIT_OK) return st;
  if ((st = check_bhnd(v)) != SAFEDIT_OK) return st;
  if ((st = check_bhnd(out)) != SAFEDIT_OK) return st;
  const int64_t B = q->dims[0], H = q->dims[1], Nq = q->dims[2], D = q->dims[3];
  const int64_t Nk = k->dims[2];
  for (const safedit_tensor* t : {k, v})
    if (t->dims[0] != B || t->dims[1] != H || t->dims[3] != D || t->dims[2] != Nk)
      return SAFEDIT_ERR_SHAPE;
  if (D != 64 && D != 96 && D != 128) return SAFEDIT_ERR_UNSUPPORTED;
  if (Nk < 1 || Nq > INT32_MAX || Nk > INT32_MAX || B * H > 65535) return SAFEDIT_ERR_SHAPE;
  if (out_scattered != 0 && out_scattered != 1) return SAFEDIT_ERR_INVALID_ARG;
  if (d_idx && n_idx < 0) return SAFEDIT_ERR_INVALID_ARG;
  const int64_t n_rows = d_idx ? n_idx : Nq;
  if ((n_rows + 255) / 256 * B * H > INT32_MAX) return SAFEDIT_ERR_SHAPE;  // units counted in int
  if (out->dims[0] != B || out->dims[1] != H || out->dims[3] != D) return SAFEDIT_ERR_SHAPE;
  if (out_scattered ? (out->dims[2] != Nq) : (out->dims[2] != n_rows)) return SAFEDIT_ERR_SHAPE;
  AttnParams p{};
  if (key_pad) {
    if ((st = check_tensor(key_pad, 2)) != SAFEDIT_OK) return st;
    if (key_pad->dtype != SAFEDIT_F32) return SAFEDIT_ERR_DTYPE;
    if (key_pad->dims[0] != B || key_pad->dims[1] != Nk) return SAFEDIT_ERR_SHAPE;
    if (key_pad->strides[1] != 1 || key_pad->strides[0] % 4 != 0 || !aligned16(key_pad->data))
      return SAFEDIT_ERR_ALIGNMENT;
    p.pad = static_cast<const float*>(key_pad->data);
    p.pad_sb = key_pad->strides[0];
  }
  if (bias) {
    if ((st = check_tensor(bias, 4)) != SAFEDIT_OK) return st;
    if (bias->dtype != SAFEDIT_F32 && bias->dtype != SAFEDIT_BF16) return SAFEDIT_ERR_DTYPE;
    if (bias->dims[0] != B || (bias->dims[1] != 1 && bias->dims[1] != H) || bias->dims[2] != Nq ||
        bias->dims[3] != Nk)
      return SAFEDIT_ERR_SHAPE;
    const int vecw = bias->dtype == SAFEDIT_F32 ? 4 : 8;
    if (bias->strides[3] != 1 || bias->strides[2] % vecw != 0 || bias->strides[1] % vecw != 0 ||
        bias->strides[0] % vecw != 0 || !aligned16(bias->data))
      return SAFEDIT_ERR_ALIGNMENT;
    p.bias = bias->data;
    p.bias_f32 = bias->dtype == SAFEDIT_F32;
    p.bias_sb = bias->strides[0];
    p.bias_sh = bias->dims[1] == 1 ? 0 : bias->strides[1];
    p.bias_sq = bias->strides[2];
  }
  AttnPlan pl = plan_attn(n_rows, B * H, Nk, int(D), use_ws, sm_count());
  if (use_ws && pl.ws_bytes > 0) {
    if (!d_ws || ws_bytes < pl.ws_bytes) return SAFEDIT_ERR_INVALID_ARG;
    if (!aligned16(d_ws)) return SAFEDIT_ERR_ALIGNMENT;
  }
  if (n_rows == 0 || B * H == 0) return SAFEDIT_OK;
  p.n_rb = pl.n_rb;
  p.n_full = pl.n_full;
  p.split = pl.split;
  p.n_part_units = pl.n_part_units;
  p.part = static_cast<float*>(d_ws);
  p.q = static_cast<const __nv_bfloat16*>(q->data);
  p.q_sb = q->strides[0];
  p.q_sh = q->strides[1];
  p.q_sr = q->strides[2];
  p.idx = d_idx;
  p.n_rows = static_cast<int>(n_rows);
  p.Nq = static_cast<int>(Nq);
  p.Nk = static_cast<int>(Nk);
  p.H = static_cast<int>(H);
  const float sc = (scale > 0.f) ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale = sc;
  p.scale_log2 = sc * kLog2e;
  p.out = static_cast<__nv_bfloat16*>(out->data);
  p.o_sb = out->strides[0];
  p.o_sh = out->strides[1];
  p.o_sr = out->strides[2];
  p.out_scattered = out_scattered;
  p.wait_limit = wait_limit_ns();
  CUtensorMap tmK, tmV;
  if ((st = make_kv_map(&tmK, k, static_cast<int>(D))) != SAFEDIT_OK) return st;
  if ((st = make_kv_map(&tmV, v, static_cast<int>(D))) != SAFEDIT_OK) return st;
  p.status = status_ptr();
  if (!p.status) return SAFEDIT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d_idx && out_scattered && index_check_enabled() &&
      (st = launch_index_check(d_idx, static_cast<int32_t>(n_rows), Nq, p.status, s)) != SAFEDIT_OK)
    return st;
  switch (D) {
    case 64: return dispatch_attn<64>(tmK, tmV, p, static_cast<int>(B), s);
    case 96: return dispatch_attn<96>(tmK, tmV, p, static_cast<int>(B), s);
    default: return dispatch_attn<128>(tmK, tmV, p, static_cast<int>(B), s);
  }
}

extern "C" safedit_status safedit_attn_subset(const safedit_tensor* q, const safedit_tensor* k,
                                              const safedit_tensor* v, const int32_t* d_idx,
                                              int32_t n_idx, const safedit_tensor* key_pad,
                                              const safedit_tensor* bias, float scale,
                                              const safedit_tensor* out, int32_t out_scattered,
                                              void* stream) {
  return attn_subset_impl(q, k, v, d_idx, n_idx, key_pad, bias, scale, out, out_scattered, nullptr, 0,
                          false, stream);
}

extern "C" safedit_status safedit_attn_subset_ws(const safedit_tensor* q, const safedit_tensor* k,
                                                 const safedit_tensor* v, const int32_t* d_idx,
                                                 int32_t n_idx, const safedit_tensor* key_pad,
                                                 const safedit_tensor* bias, float scale,
                                                 const safedit_tensor* out, int32_t out_scattered,
                                                 void* d_workspace, size_t workspace_bytes,
                                                 void* stream) {
  return attn_subset_impl(q, k, v, d_idx, n_idx, key_pad, bias, scale, out, out_scattered, d_workspace,
                          workspace_bytes, true, stream);
}

extern "C" size_t safedit_attn_subset_workspace_size(int64_t batch, int64_t heads, int64_t n_rows,
                                                     int64_t n_keys, int32_t head_dim) {
  if (batch <= 0 || heads <= 0 || n_rows <= 0 || n_keys <= 0) return 0;
  if (head_dim != 64 && head_dim != 96 && head_dim != 128) return 0;
  if (batch * heads > 65535 || n_rows > INT32_MAX || n_keys > INT32_MAX ||
      (n_rows + 255) / 256 * batch * heads > INT32_MAX)
    return 0;
  return plan_attn(n_rows, batch * heads, n_keys, head_dim, true, sm_count()).ws_bytes;
}
