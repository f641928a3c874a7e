/*
 * safedit.h -- C ABI of libsafedit.so: the mask-free spatially adaptive DiT
 * attention path on one NVIDIA B200 (sm_100a).
 *
 * The method (SAFE-DiT, and AccelAes' SkipSparse) is described on:
 *   [P1] "기술 요약: SAFE-DiT" (gist.science/ko/paper/2606.29360), 방법론 1-4;
 *   [P4] "SAFE-DiT: Semantics-Aware Fast-path Execution for High-Resolution
 *        Diffusion Transformers" (gist.science/it/paper/2606.29360),
 *        Metodologia 1-4 (same content);
 *   [P3] AccelAes technical summary (gist.science/ko/paper/2603.12575),
 *        방법론 B.1 (AesMask) and B.2 (SkipSparse).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Memory.  Every pointer named d_* and every safedit_tensor.data is DEVICE
 *   memory on the current CUDA device; host_* pointers are host memory.  The
 *   caller owns and allocates every buffer.  The library allocates nothing
 *   except one static device status word per device and the static scratch
 *   array of safedit_attn_subset_noalloc (both reserved when the library's
 *   device code loads, never at call time).  A pointer to an array
 *   with no elements (an empty tensor, a zero-length vector) may be NULL.
 * - Empty work.  A call whose work is empty (no rows, no tokens, no
 *   columns) checks its arguments, launches nothing and returns SAFEDIT_OK.
 * - Streams.  `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   Every call only enqueues work on that stream and returns without
 *   synchronising, except safedit_get_device_status.
 * - Errors.  Argument errors are detected on the host and returned before
 *   any launch (at most the current device and its attributes are read).
 *   Errors found on the device
 *   (an index out of range, a fully masked row, a pipeline wait that timed
 *   out) set the device status word, which safedit_get_device_status reads
 *   and clears; the outputs of the failing call are then unspecified.
 * - Layout.  safedit_tensor gives dims and element strides (not bytes), outer
 *   to inner.  Attention tensors are [B, H, rows, d] with d contiguous
 *   (strides[3] == 1) and every other stride a multiple of 8 elements
 *   (16 bytes); data must be 16-byte aligned.
 * - Threading.  Stateless and reentrant apart from the status word, the
 *   launch counter, the debug settings (wait limit, index check) and the
 *   scratch array of safedit_attn_subset_noalloc, which calls that overlap
 *   on one device share.
 */
#ifndef SAFEDIT_H_
#define SAFEDIT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAFEDIT_OK = 0,
  SAFEDIT_ERR_INVALID_ARG = 1, /* null pointer, bad enum, bad count        */
  SAFEDIT_ERR_SHAPE = 2,       /* dims that do not agree                   */
  SAFEDIT_ERR_DTYPE = 3,       /* element type not supported by the call   */
  SAFEDIT_ERR_ALIGNMENT = 4,   /* pointer or stride not 16-byte aligned    */
  SAFEDIT_ERR_INDEX = 5,       /* index out of range (device-detected)     */
  SAFEDIT_ERR_UNSUPPORTED = 6, /* e.g. a head dim other than 64/96/128     */
  SAFEDIT_ERR_CUDA = 7,        /* a CUDA runtime/driver call failed        */
  SAFEDIT_ERR_TIMEOUT = 8,     /* a bounded on-device wait gave up         */
  SAFEDIT_ERR_MASKED_ROW = 9   /* a row with no admissible key (device)    */
} safedit_status;

typedef enum {
  SAFEDIT_F32 = 0,
  SAFEDIT_BF16 = 1,
  SAFEDIT_F16 = 2,
  SAFEDIT_BOOL = 3, /* one byte, nonzero = true */
  SAFEDIT_I32 = 4,
  SAFEDIT_F64 = 5,
  SAFEDIT_U8 = 6
} safedit_dtype;

typedef struct {
  void *data;         /* device pointer to element [0,0,...]          */
  int32_t dtype;      /* safedit_dtype                                */
  int32_t ndim;       /* 1..4                                         */
  int64_t dims[4];    /* outer to inner; only the first ndim are read */
  int64_t strides[4]; /* element strides; 0 marks a broadcast dim     */
} safedit_tensor;

/* ------------------------------------------------------------------------
 * PCSP score producer: image->text cross-attention probabilities.
 * [P1 방법론 2 / P4 Metodologia 2]: in a short warm-up the attention weights
 * from image tokens to text content tokens are gathered; [P3 B.1 step 3].
 * [P1 방법론 1 보존]: text padding stays masked, so padding keys get exactly 0.
 *
 *   P[h,i,j] = softmax_j( scale * q_img[b,h,i,:] . k_txt[b,h,j,:] )
 * over the keys with d_key_valid[b*L + j] != 0 (b = batch_index), and
 * P[h,i,j] = 0 exactly for the others.
 *
 * q_img  [B,H,N,d] bf16, d in {64,96,128}.     k_txt [B,H,L,d] bf16, L <= 256.
 * d_key_valid [B*L] u8 (row-major [B,L]).      scale: 0 selects 1/sqrt(d).
 * p_out  [H,N,L] f32, strides {N*L', L', 1} with L' >= L, L' % 4 == 0.
 * A row with no valid key sets SAFEDIT_ERR_MASKED_ROW and writes zeros.
 */
safedit_status safedit_cross_attn_probs(const safedit_tensor *q_img,
                                        const safedit_tensor *k_txt,
                                        const uint8_t *d_key_valid,
                                        int32_t batch_index, float scale,
                                        const safedit_tensor *p_out,
                                        void *stream);

/* ------------------------------------------------------------------------
 * PCSP aggregation.  [P1 방법론 2 / P4 Metodologia 2]; [P3 B.1 step 3].
 *
 *   d_score[i] += sum_h sum_{j : d_content[j] != 0} P[h,i,j]
 * accumulated in fp64.  Call it once per warm-up step (and layer) with the
 * same score buffer; zero the buffer before the first call.
 *
 * p [H,N,L] f32 or bf16 (widened exactly), inner stride 1.  d_content [L]
 * u8.  d_score [N] f64.
 */
safedit_status safedit_partition_accumulate(const safedit_tensor *p,
                                            const uint8_t *d_content,
                                            double *d_score, void *stream);

/* ------------------------------------------------------------------------
 * PCSP split into the sensitive set S and the context set C, plus the
 * sensitivity score s.  [P1 방법론 2, 4 / P4 Metodologia 2, 4]: the split is
 * fixed for the whole trajectory; s_i drives the per-token guidance scale.
 * [P3 B.1 step 4]: a percentile threshold, here a top-k by count.
 *
 * S = the k tokens of largest score, ties to the lower index; d_idx_s [k]
 * and d_idx_c [n-k] are written in ascending token order.  d_s [n] (nullable)
 * gets (score - min) / (max - min) computed in fp64 and rounded to f32, or 0
 * when all scores are equal.  d_idx_s / d_idx_c may be NULL to skip them.
 * 0 <= k <= n <= 1<<24.  A NaN score sets SAFEDIT_ERR_INVALID_ARG on device.
 */
safedit_status safedit_partition_finalize(const double *d_score, int32_t n,
                                          int32_t k, int32_t *d_idx_s,
                                          int32_t *d_idx_c, float *d_s,
                                          void *stream);

/* ------------------------------------------------------------------------
 * Fused PCSP score: cross-attention probabilities and their aggregation in
 * one pass, without materialising P.  [P1 방법론 2 / P4 Metodologia 2];
 * [P3 B.1 step 3].  Same result as safedit_cross_attn_probs followed by
 * safedit_partition_accumulate (up to fp32 rounding of the probabilities):
 *
 *   d_score[i] += sum_h ( sum_{j valid, content} e_hij / sum_{j valid} e_hij ),
 *   e_hij = exp(scale q_img[b,h,i,:] . k_txt[b,h,j,:] - max_j(...)),  b = batch_index.
 *
 * q_img [B,H,N,d] bf16, d in {64,96,128}; k_txt [B,H,L,d] bf16, L <= 256;
 * d_key_valid [B*L] u8; d_content [L] u8; d_score [N] f64 (in/out, fp64
 * accumulation, each row's heads summed inside one CTA: deterministic).
 * scale: 0 selects 1/sqrt(d).  A row with no valid key sets
 * SAFEDIT_ERR_MASKED_ROW and adds nothing.
 */
safedit_status safedit_pcsp_score(const safedit_tensor *q_img,
                                  const safedit_tensor *k_txt,
                                  const uint8_t *d_key_valid,
                                  const uint8_t *d_content, int32_t batch_index,
                                  float scale, double *d_score, void *stream);

/* ------------------------------------------------------------------------
 * Exact mask-elision criterion.  [P1 방법론 1 / P4 Metodologia 1]: an additive
 * mask whose effect on the logits is a per-row constant c_i (L_{i,:} + c_i)
 * leaves softmax unchanged and may be removed; text padding, causal and
 * non-uniform bias masks are kept.
 *
 * mask [B, Hm, Nq, Nk] (ndim 2..4; missing outer dims are 1) in f32, bf16,
 * f16 (additive) or bool (true = attend = 0, false = -inf); strides may be 0
 * for broadcast dims; inner stride 1 or 0.  A row is removable iff all its
 * entries equal entry 0 (IEEE ==: +0 == -0, NaN never) and that entry is
 * finite.  *d_verdict (i32) = 1 if every row is removable, else 0.
 * d_row_flags (nullable) [B*Hm*Nq] u8 row-major = per-row verdicts; when it
 * is NULL the kernel may stop reading once a kept row is found.
 */
safedit_status safedit_mask_is_row_constant(const safedit_tensor *mask,
                                            int32_t *d_verdict,
                                            uint8_t *d_row_flags,
                                            void *stream);

/* ------------------------------------------------------------------------
 * SRSU subset attention and CAR dense anchor.  [P1 방법론 3 / P4
 * Metodologia 3]: on non-anchor steps only the query rows of S are updated,
 * and they attend over the global keys/values (fresh S states + cached C
 * states); anchor steps refresh every row densely.  [P3 B.2]: queries only
 * on focus tokens, keys and values from the whole image.
 *
 * For r in [0, n_rows), i = d_idx[r] (i = r when d_idx is NULL):
 *   out_r = sum_j softmax_j( scale * q[b,h,i,:] . k[b,h,j,:]
 *                            + key_pad[b,j] + bias[b,h',i,j] ) v[b,h,j,:]
 * over all Nk keys, fp32 accumulation, bf16 result.
 *
 * q [B,H,Nq,d] bf16; k, v [B,H,Nk,d] bf16; d in {64, 96, 128}.
 * d_idx [n_idx] i32 in [0, Nq) and unique, or NULL (then n_rows = Nq and
 *   n_idx is ignored).  Out-of-range indices set SAFEDIT_ERR_INDEX and the
 *   row is skipped.  Uniqueness is the caller's contract (the split of
 *   safedit_partition_finalize is unique by construction); with
 *   out_scattered == 1 and the debug index check on, a duplicate sets
 *   SAFEDIT_ERR_INDEX (see safedit_debug_set_index_check).
 * key_pad (nullable) [B, Nk] f32, additive (0 or -inf for kept text padding);
 *   inner stride 1, batch stride a multiple of 4 elements, data 16-byte
 *   aligned.  Key tiles of 128 keys whose pad is -inf throughout carry exactly
 *   zero weight and are not computed (an exact shortcut).
 * bias (nullable) [B, 1|H, Nq, Nk] f32 or bf16, additive, a kept non-uniform
 *   bias; inner stride 1, every other stride a multiple of 16 bytes (4 f32 or
 *   8 bf16 elements), data 16-byte aligned.
 * scale: 0 selects 1/sqrt(d).
 * out: out_scattered == 0 -> [B,H,n_rows,d] compact (row r at r);
 *      out_scattered == 1 -> [B,H,Nq,d] state, row r written at index i
 *      (rows not in d_idx are left untouched).  bf16.
 * A row whose every key is masked sets SAFEDIT_ERR_MASKED_ROW and gets zeros.
 */
safedit_status safedit_attn_subset(const safedit_tensor *q,
                                   const safedit_tensor *k,
                                   const safedit_tensor *v,
                                   const int32_t *d_idx, int32_t n_idx,
                                   const safedit_tensor *key_pad,
                                   const safedit_tensor *bias, float scale,
                                   const safedit_tensor *out,
                                   int32_t out_scattered, void *stream);

/* ------------------------------------------------------------------------
 * The same attention with the tail of the launch balanced over the SMs (a
 * scheduling choice of this library: the pages define only the result,
 * the SRSU rows over all keys of [P1 방법론 3]).  The work is cut into
 * units of 256 query rows of one (b, h) slice.  When the units do not fill
 * the last wave of the GPU's SMs, each of those last units may run as
 * s = 2..4 parts over the key tiles: the whole units run first as one
 * launch (a whole number of waves), the parts as a second launch that may
 * start while the first one's last wave drains (programmatic dependent
 * launch; it completes only after the first), writing their unnormalised
 * output rows, running max and row sum (f32) to d_workspace, and a merge
 * kernel then combines them into the output rows (the online-softmax merge;
 * the result equals safedit_attn_subset's within the attention tolerance,
 * not bit for bit).  Kept masks (key_pad, bias) are split like the rest;
 * a part whose key range holds no admissible key for a row leaves it to
 * the merge, which reports a row with none in any part as
 * SAFEDIT_ERR_MASKED_ROW and writes zeros, as safedit_attn_subset does.
 * The plan takes a split only where a per-CTA cost model (set-up +
 * per-key-tile time of the mask-free kernel, measured on B200) predicts a
 * saving of at least 3% of the call; otherwise the call is
 * safedit_attn_subset.  All launches go on `stream`, in order, so the call
 * is stream-ordered like the others.
 *
 * Arguments as safedit_attn_subset, plus d_workspace / workspace_bytes:
 * device memory of at least safedit_attn_subset_workspace_size(...) bytes
 * for this call on the current device, 16-byte aligned (else
 * SAFEDIT_ERR_ALIGNMENT), owned by the caller, not read before it is
 * written; NULL is allowed when that size is 0.  A smaller workspace returns
 * SAFEDIT_ERR_INVALID_ARG before any launch.  Calls that share a workspace
 * must not overlap on the GPU.
 */
safedit_status safedit_attn_subset_ws(const safedit_tensor *q,
                                      const safedit_tensor *k,
                                      const safedit_tensor *v,
                                      const int32_t *d_idx, int32_t n_idx,
                                      const safedit_tensor *key_pad,
                                      const safedit_tensor *bias, float scale,
                                      const safedit_tensor *out,
                                      int32_t out_scattered,
                                      void *d_workspace, size_t workspace_bytes,
                                      void *stream);

/* Workspace bytes safedit_attn_subset_ws needs on the current device (its
 * SM count enters the plan) for batch x heads slices of n_rows query rows
 * over n_keys keys of head_dim (64, 96 or 128): (split units) x s x 256 x
 * (head_dim + 2) x 4, with or without kept masks; 0 when the plan keeps
 * whole units.  Host only, no launch; invalid sizes give 0. */
size_t safedit_attn_subset_workspace_size(int64_t batch, int64_t heads,
                                          int64_t n_rows, int64_t n_keys,
                                          int32_t head_dim);

/* ------------------------------------------------------------------------
 * safedit_attn_subset_ws without a caller workspace.  The pages have no
 * counterpart: this is a deployment variant for callers that may not
 * allocate device memory around the call, not a step of the method.
 *
 * Arguments and result as safedit_attn_subset_ws.  The workspace is a
 * fixed array of SAFEDIT_ATTN_NOALLOC_SCRATCH_BYTES (24 MiB) per device
 * inside the library, reserved when its device code is loaded; the call
 * allocates nothing.  A call whose plan needs more
 * (safedit_attn_subset_workspace_size(...) > the limit) returns
 * SAFEDIT_ERR_UNSUPPORTED before any launch.  The first call on a device
 * (with that device current) looks the array's address up
 * (cudaGetSymbolAddress) and caches it: make that first call before any
 * stream capture.  Nothing in the array needs to start at zero (the parts
 * write their results in full before the merge reads them), so nothing is
 * cleared.  All calls on one device share the array: calls that overlap
 * on the GPU (other streams, other host threads) race on it.
 */
#define SAFEDIT_ATTN_NOALLOC_SCRATCH_BYTES ((size_t)24 << 20)

safedit_status safedit_attn_subset_noalloc(const safedit_tensor *q,
                                           const safedit_tensor *k,
                                           const safedit_tensor *v,
                                           const int32_t *d_idx, int32_t n_idx,
                                           const safedit_tensor *key_pad,
                                           const safedit_tensor *bias,
                                           float scale,
                                           const safedit_tensor *out,
                                           int32_t out_scattered, void *stream);

/* ------------------------------------------------------------------------
 * State scatter.  [P1 방법론 3 / P4 Metodologia 3]: context states are cached
 * and reused between anchors; fresh sensitive rows replace their entries.
 *
 * For t < n_tensors: dst[t][b,h,d_idx[r],:] = src[t][b,h,r,:], r < n_idx.
 * src[t] [B,H,n_idx,d], dst[t] [B,H,N,d], same dtype (any 2- or 4-byte
 * type), same B, H, d per pair; d*elt % 16 == 0.  1 <= n_tensors <= 4, one
 * launch for all.  d_idx must be unique: two equal entries would race for
 * one row (checked only in the debug index-check mode, where a duplicate
 * sets SAFEDIT_ERR_INDEX); out-of-range entries set SAFEDIT_ERR_INDEX and
 * are skipped.  Other rows are untouched.
 */
safedit_status safedit_scatter_state(const safedit_tensor *src,
                                     const safedit_tensor *dst,
                                     int32_t n_tensors, const int32_t *d_idx,
                                     int32_t n_idx, void *stream);

/* Gather, the inverse: dst[t][b,h,r,:] = src[t][b,h,d_idx[r],:]. */
safedit_status safedit_gather_rows(const safedit_tensor *src,
                                   const safedit_tensor *dst,
                                   int32_t n_tensors, const int32_t *d_idx,
                                   int32_t n_idx, void *stream);

/* ------------------------------------------------------------------------
 * Sensitivity-weighted CFG.  [P1 방법론 4 / P4 Metodologia 4]:
 *   gamma_i = gamma_ctx + (gamma_sens - gamma_ctx) * s_i,
 * applied to the prediction after the forward pass; [P3 B.2] spatial CFG.
 *   out[i,f] = eps_u[i,f] + gamma_i * (eps_c[i,f] - eps_u[i,f])   (f32 FMA)
 * eps_c, eps_u [N, F] f32, or both bf16 (widened exactly to f32), with
 * inner stride 1; out [N, F] f32, inner stride 1 (with f32 inputs out may
 * alias either input; with bf16 inputs it must not overlap them).  d_s [N]
 * f32.  gamma_ctx == gamma_sens gives plain CFG (SAFE-Core).
 */
safedit_status safedit_sw_cfg(const safedit_tensor *eps_c,
                              const safedit_tensor *eps_u, const float *d_s,
                              float gamma_ctx, float gamma_sens,
                              const safedit_tensor *out, void *stream);

/* ------------------------------------------------------------------------
 * StepCache with sensitivity-weighted CFG.  [P3 B.3]: full inference runs
 * only every Delta steps and the noise prediction is reused in between by
 * linear extrapolation; combined here with the guidance of [P1 방법론 4]:
 *   c = c_b + w (c_b - c_a),   u = u_b + w (u_b - u_a),
 *   out = u + gamma_i (c - u),  gamma_i = gamma_ctx + (gamma_sens - gamma_ctx) s_i
 * where a, b are the last two full steps (b later) and w = (t - t_b)/(t_b - t_a).
 * All tensors [N, F] f32, inner stride 1 (out may alias an input); d_s [N] f32.
 */
safedit_status safedit_stepcache_sw_cfg(const safedit_tensor *eps_c_a,
                                        const safedit_tensor *eps_c_b,
                                        const safedit_tensor *eps_u_a,
                                        const safedit_tensor *eps_u_b,
                                        const float *d_s, float w,
                                        float gamma_ctx, float gamma_sens,
                                        const safedit_tensor *out, void *stream);

/* ------------------------------------------------------------------------
 * Dense projection with fused bias and activation, and optional row scatter:
 * the GEMM of SkipSparse FFN caching [P3 B.2], where the FFN runs on the
 * sensitive (focus) tokens only and every other token keeps its cached FFN
 * output.  With X_S the gathered sensitive rows:
 *   H   = GELU(X_S W1^T + b1)                       (act = 1, d_idx_out NULL)
 *   Y[idx[r], :] = (H W2^T + b2)[r, :]             (act = 0, d_idx_out = idx)
 * and the same call with act = 0 serves the gathered Q/K/V projections.
 *
 *   out[row(r), n] = act( sum_k a[r,k] * w[n,k] + bias[n] ),  r < M, n < N
 *   row(r) = d_idx_out ? d_idx_out[r] : r
 *
 * a [M, K] or batched [B, M, K], w [N, K] (nn.Linear layout: out_features x
 * in_features), bf16, inner stride 1, row and batch strides multiples of 8
 * elements, 16-byte aligned bases.  out [M_out, N] or [B, M_out, N] (same
 * rank as a, same rules); w and d_idx_out are shared by every batch; without
 * d_idx_out M_out must equal M.  N must be a multiple of 8.  d_bias: NULL or
 * N f32 on the device.  act: 0 identity, 1 GELU (tanh form, fp32).
 * Accumulation is fp32 over all of K (tensor cores), rounded to bf16 once.
 * d_idx_out: NULL or M int32 on the device, unique (checked only in the
 * debug index-check mode, where a duplicate sets SAFEDIT_ERR_INDEX); an entry
 * outside [0, M_out) sets SAFEDIT_ERR_INDEX on the device status word and
 * that row is skipped.  Rows of out that no r maps to are untouched.
 * M == 0 or N == 0 is a no-op; K == 0 is SAFEDIT_ERR_SHAPE.
 */
safedit_status safedit_gemm_bias_act(const safedit_tensor *a,
                                     const safedit_tensor *w,
                                     const float *d_bias, int32_t act,
                                     const int32_t *d_idx_out,
                                     const safedit_tensor *out, void *stream);

/* ------------------------------------------------------------------------
 * Device status word: on `stream`, takes the word of the current device out
 * and clears it in one atomic step (a one-thread kernel), then waits for the
 * stream and stores it in *host_status (a safedit_status value, SAFEDIT_OK if
 * nothing was flagged since the last read).  An error that a kernel on
 * another stream records meanwhile is either returned by this call or kept
 * for the next one.
 */
safedit_status safedit_get_device_status(int32_t *host_status, void *stream);

/* Static English text of a status code (never NULL). */
const char *safedit_status_string(safedit_status status);

/* Number of kernels this library has launched in this process (monotone). */
uint64_t safedit_kernel_launch_count(void);

/* Debug knob: limit, in nanoseconds, for every bounded spin-wait inside the
 * pipelined kernels (default 1e9).  0 makes the first wait that is not
 * already satisfied give up, which exercises the SAFEDIT_ERR_TIMEOUT path
 * without a real hang.  Returns the previous value. */
uint64_t safedit_debug_set_wait_limit_ns(uint64_t ns);

/* Debug knob: with `on` non-zero, every call that writes rows through an
 * index vector (safedit_scatter_state, safedit_attn_subset with
 * out_scattered == 1, safedit_gemm_bias_act with d_idx_out) first launches a
 * check of that vector on the same stream: an entry out of range or equal to
 * an earlier one sets SAFEDIT_ERR_INDEX in the device status word (the
 * scattering kernel still runs; its output is then unspecified).  The check
 * is one CTA with a bitmap of the row range in shared memory and allocates
 * nothing.  Off by default.  Returns the previous setting. */
int32_t safedit_debug_set_index_check(int32_t on);

#ifdef __cplusplus
}
#endif

#endif /* SAFEDIT_H_ */
