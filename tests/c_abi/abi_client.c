/* A plain C client of libsafedit.so (include/safedit.h), with no Python in
 * the loop: device memory from the CUDA runtime, seeded inputs from a small
 * LCG, one SRSU subset-attention call (gathered rows over all keys, output
 * scattered into a state), the same rows through the tail-balanced entry
 * points (a caller workspace, and the library's fixed array), the same rows
 * with kept masks (key padding and an f32 bias, compact output), one
 * row-constant mask check and one SW-CFG call, each compared with the fp64
 * oracle (test infrastructure, liboracle.so).
 *
 *   abi_client          run the checks on the current CUDA device (exit 0 = pass)
 *   abi_client --abi    only the host-side argument checks (no GPU needed)
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "safedit.h"

/* oracle entry points (fp64, tests only) */
int oracle_attn_subset(int64_t Nq, int64_t N, int64_t d, const double *q, const double *k,
                       const double *v, const int32_t *idx, int64_t n_idx, const double *pad,
                       const double *bias_rows, double scale, double *out);
void oracle_sw_cfg(int64_t N, int64_t F, const double *eps_c, const double *eps_u,
                   const double *s, double gamma_ctx, double gamma_sens, double *out);

static uint64_t lcg_state = 0x5eed5afeull;
static double uniform01(void) { /* 53-bit uniform in [0, 1) */
  lcg_state = lcg_state * 6364136223846793005ull + 1442695040888963407ull;
  return (double)(lcg_state >> 11) * (1.0 / 9007199254740992.0);
}
static double normal01(void) { /* Box-Muller */
  double u1 = uniform01(), u2 = uniform01();
  if (u1 < 1e-300) u1 = 1e-300;
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}
/* float -> bf16 bits, round to nearest even (finite inputs) */
static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static double from_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

#define CHECK_CUDA(x)                                                     \
  do {                                                                    \
    cudaError_t e_ = (x);                                                 \
    if (e_ != cudaSuccess) {                                              \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));            \
      return 2;                                                           \
    }                                                                     \
  } while (0)
#define CHECK_SD(x)                                                       \
  do {                                                                    \
    safedit_status s_ = (x);                                              \
    if (s_ != SAFEDIT_OK) {                                               \
      fprintf(stderr, "%s: %s\n", #x, safedit_status_string(s_));         \
      return 3;                                                           \
    }                                                                     \
  } while (0)

static safedit_tensor tensor4(void *data, safedit_dtype dt, int64_t a, int64_t b, int64_t c,
                              int64_t d) {
  safedit_tensor t;
  memset(&t, 0, sizeof t);
  t.data = data;
  t.dtype = dt;
  t.ndim = 4;
  t.dims[0] = a, t.dims[1] = b, t.dims[2] = c, t.dims[3] = d;
  t.strides[3] = 1, t.strides[2] = d, t.strides[1] = c * d, t.strides[0] = b * c * d;
  return t;
}

/* host-side argument checks: nothing is launched, no GPU is touched */
static int abi_checks(void) {
  int bad = 0;
  uint64_t n0 = safedit_kernel_launch_count();
  safedit_tensor q = tensor4((void *)256, SAFEDIT_BF16, 1, 1, 64, 80); /* d = 80 */
  if (safedit_attn_subset(&q, &q, &q, NULL, 0, NULL, NULL, 0.f, &q, 0, NULL) !=
      SAFEDIT_ERR_UNSUPPORTED)
    bad = 1;
  safedit_tensor f = tensor4((void *)256, SAFEDIT_F32, 1, 1, 64, 64);
  if (safedit_attn_subset(&f, &f, &f, NULL, 0, NULL, NULL, 0.f, &f, 0, NULL) != SAFEDIT_ERR_DTYPE)
    bad = 1;
  if (safedit_partition_finalize(NULL, 10, 11, NULL, NULL, NULL, NULL) != SAFEDIT_ERR_INVALID_ARG)
    bad = 1;
  if (safedit_kernel_launch_count() != n0) bad = 1;
  if (strcmp(safedit_status_string(SAFEDIT_OK), "ok") != 0) bad = 1;
  printf("abi checks: %s\n", bad ? "FAILED" : "ok");
  return bad;
}

int main(int argc, char **argv) {
  if (argc > 1 && strcmp(argv[1], "--abi") == 0) return abi_checks();
  if (abi_checks()) return 1;

  /* one (b, h) slice: N = 1100 keys and queries (9 key tiles), d = 96, 330
   * gathered rows (2 units of 256 rows) */
  const int64_t N = 1100, d = 96, n_idx = 330;
  const size_t nel = (size_t)(N * d);
  uint16_t *hq = malloc(nel * 2), *hk = malloc(nel * 2), *hv = malloc(nel * 2), *ho = malloc(nel * 2);
  double *q = malloc(nel * 8), *k = malloc(nel * 8), *v = malloc(nel * 8);
  double *ref = malloc((size_t)(n_idx * d) * 8);
  int32_t *idx = malloc((size_t)n_idx * 4);
  if (!hq || !hk || !hv || !ho || !q || !k || !v || !ref || !idx) return 2;
  for (size_t i = 0; i < nel; ++i) {
    hq[i] = to_bf16((float)normal01());
    hk[i] = to_bf16((float)normal01());
    hv[i] = to_bf16((float)normal01());
    q[i] = from_bf16(hq[i]), k[i] = from_bf16(hk[i]), v[i] = from_bf16(hv[i]);
    ho[i] = 0x3F80u; /* 1.0: rows outside idx must keep it */
  }
  for (int64_t r = 0; r < n_idx; ++r) idx[r] = (int32_t)(r * 10 / 3); /* ascending, unique */

  void *dq, *dk, *dv, *dout, *didx;
  CHECK_CUDA(cudaMalloc(&dq, nel * 2));
  CHECK_CUDA(cudaMalloc(&dk, nel * 2));
  CHECK_CUDA(cudaMalloc(&dv, nel * 2));
  CHECK_CUDA(cudaMalloc(&dout, nel * 2));
  CHECK_CUDA(cudaMalloc(&didx, (size_t)n_idx * 4));
  CHECK_CUDA(cudaMemcpy(dq, hq, nel * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dk, hk, nel * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dv, hv, nel * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dout, ho, nel * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(didx, idx, (size_t)n_idx * 4, cudaMemcpyHostToDevice));

  safedit_tensor tq = tensor4(dq, SAFEDIT_BF16, 1, 1, N, d);
  safedit_tensor tk = tensor4(dk, SAFEDIT_BF16, 1, 1, N, d);
  safedit_tensor tv = tensor4(dv, SAFEDIT_BF16, 1, 1, N, d);
  safedit_tensor to = tensor4(dout, SAFEDIT_BF16, 1, 1, N, d);
  CHECK_SD(safedit_attn_subset(&tq, &tk, &tv, (const int32_t *)didx, (int32_t)n_idx, NULL, NULL,
                               0.f, &to, 1, NULL));
  int32_t status = -1;
  CHECK_SD(safedit_get_device_status(&status, NULL));
  if (status != SAFEDIT_OK) {
    fprintf(stderr, "device status %s\n", safedit_status_string((safedit_status)status));
    return 4;
  }
  CHECK_CUDA(cudaMemcpy(ho, dout, nel * 2, cudaMemcpyDeviceToHost));
  if (oracle_attn_subset(N, N, d, q, k, v, idx, n_idx, NULL, NULL, 1.0 / sqrt((double)d), ref) != 0)
    return 5;
  double num = 0.0, den = 0.0, mx = 0.0;
  for (int64_t r = 0; r < n_idx; ++r)
    for (int64_t c = 0; c < d; ++c) {
      const double g = from_bf16(ho[(size_t)idx[r] * d + c]), e = ref[r * d + c];
      num += (g - e) * (g - e), den += e * e;
      if (fabs(g - e) > mx) mx = fabs(g - e);
    }
  const double rel = sqrt(num / den);
  int kept = 1;
  for (int64_t i = 0, r = 0; i < N; ++i) {
    if (r < n_idx && idx[r] == i) {
      ++r;
      continue;
    }
    for (int64_t c = 0; c < d; ++c) kept &= ho[(size_t)i * d + c] == 0x3F80u;
  }
  printf("attn_subset: relFro %.3e  max|err| %.3e  untouched rows %s\n", rel, mx,
         kept ? "ok" : "CHANGED");
  if (!(rel <= 5e-3 && mx <= 2e-2 && kept)) return 6;

  /* the same call through the tail-balanced entry points: both units run as
   * key-range parts merged afterwards, the partial results first in a
   * caller workspace, then in the library's fixed array */
  const size_t ws_bytes = safedit_attn_subset_workspace_size(1, 1, n_idx, N, (int32_t)d);
  if (ws_bytes == 0) return 11;
  void *dws;
  CHECK_CUDA(cudaMalloc(&dws, ws_bytes));
  for (int variant = 0; variant < 2; ++variant) {
    CHECK_CUDA(cudaMemset(dout, 0, nel * 2));
    if (variant == 0)
      CHECK_SD(safedit_attn_subset_ws(&tq, &tk, &tv, (const int32_t *)didx, (int32_t)n_idx, NULL, NULL,
                                      0.f, &to, 1, dws, ws_bytes, NULL));
    else
      CHECK_SD(safedit_attn_subset_noalloc(&tq, &tk, &tv, (const int32_t *)didx, (int32_t)n_idx, NULL,
                                           NULL, 0.f, &to, 1, NULL));
    CHECK_SD(safedit_get_device_status(&status, NULL));
    if (status != SAFEDIT_OK) {
      fprintf(stderr, "device status %s\n", safedit_status_string((safedit_status)status));
      return 4;
    }
    CHECK_CUDA(cudaMemcpy(ho, dout, nel * 2, cudaMemcpyDeviceToHost));
    double n2 = 0.0, d2 = 0.0, m2 = 0.0;
    for (int64_t r = 0; r < n_idx; ++r)
      for (int64_t c = 0; c < d; ++c) {
        const double g = from_bf16(ho[(size_t)idx[r] * d + c]), e = ref[r * d + c];
        n2 += (g - e) * (g - e), d2 += e * e;
        if (fabs(g - e) > m2) m2 = fabs(g - e);
      }
    printf("%s (%zu-byte partials): relFro %.3e  max|err| %.3e\n",
           variant == 0 ? "attn_subset_ws" : "attn_subset_noalloc", ws_bytes, sqrt(n2 / d2), m2);
    if (!(sqrt(n2 / d2) <= 5e-3 && m2 <= 2e-2)) return 12;
  }
  CHECK_CUDA(cudaFree(dws));

  /* the same rows with kept masks, compact output: a key-padding vector (key
   * tile 2 -inf throughout, so it is skipped, plus scattered -inf keys) and a
   * dense f32 bias [1,1,N,N] */
  float *hpad = malloc((size_t)N * 4), *hbias = malloc((size_t)(N * N) * 4);
  double *pad64 = malloc((size_t)N * 8), *brows = malloc((size_t)(n_idx * N) * 8);
  double *ref2 = malloc((size_t)(n_idx * d) * 8);
  uint16_t *ho2 = malloc((size_t)(n_idx * d) * 2);
  if (!hpad || !hbias || !pad64 || !brows || !ref2 || !ho2) return 2;
  for (int64_t j = 0; j < N; ++j) {
    hpad[j] = ((j >= 256 && j < 384) || j % 11 == 5) ? -INFINITY : 0.f;
    pad64[j] = hpad[j];
  }
  for (int64_t i = 0; i < N * N; ++i) hbias[i] = (float)(0.5 * normal01());
  for (int64_t r = 0; r < n_idx; ++r)
    for (int64_t j = 0; j < N; ++j) brows[r * N + j] = hbias[(int64_t)idx[r] * N + j];
  void *dpad, *dbias, *dout2;
  CHECK_CUDA(cudaMalloc(&dpad, (size_t)N * 4));
  CHECK_CUDA(cudaMalloc(&dbias, (size_t)(N * N) * 4));
  CHECK_CUDA(cudaMalloc(&dout2, (size_t)(n_idx * d) * 2));
  CHECK_CUDA(cudaMemcpy(dpad, hpad, (size_t)N * 4, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dbias, hbias, (size_t)(N * N) * 4, cudaMemcpyHostToDevice));
  safedit_tensor tpad;
  memset(&tpad, 0, sizeof tpad);
  tpad.data = dpad, tpad.dtype = SAFEDIT_F32, tpad.ndim = 2;
  tpad.dims[0] = 1, tpad.dims[1] = N, tpad.strides[0] = N, tpad.strides[1] = 1;
  safedit_tensor tbias = tensor4(dbias, SAFEDIT_F32, 1, 1, N, N);
  safedit_tensor to2 = tensor4(dout2, SAFEDIT_BF16, 1, 1, n_idx, d);
  CHECK_SD(safedit_attn_subset(&tq, &tk, &tv, (const int32_t *)didx, (int32_t)n_idx, &tpad, &tbias,
                               0.f, &to2, 0, NULL));
  CHECK_SD(safedit_get_device_status(&status, NULL));
  if (status != SAFEDIT_OK) {
    fprintf(stderr, "device status %s\n", safedit_status_string((safedit_status)status));
    return 4;
  }
  CHECK_CUDA(cudaMemcpy(ho2, dout2, (size_t)(n_idx * d) * 2, cudaMemcpyDeviceToHost));
  if (oracle_attn_subset(N, N, d, q, k, v, idx, n_idx, pad64, brows, 1.0 / sqrt((double)d), ref2) != 0)
    return 5;
  num = 0.0, den = 0.0, mx = 0.0;
  for (int64_t i = 0; i < n_idx * d; ++i) {
    const double g = from_bf16(ho2[i]), e = ref2[i];
    num += (g - e) * (g - e), den += e * e;
    if (fabs(g - e) > mx) mx = fabs(g - e);
  }
  const double rel2 = sqrt(num / den);
  printf("attn_subset with kept masks: relFro %.3e  max|err| %.3e\n", rel2, mx);
  if (!(rel2 <= 5e-3 && mx <= 2e-2)) return 10;

  /* mask check: a per-row constant additive mask [1,1,64,256] f32 is removable */
  const int64_t mq = 64, mk = 256;
  float *hm = malloc((size_t)(mq * mk) * 4);
  for (int64_t i = 0; i < mq; ++i)
    for (int64_t j = 0; j < mk; ++j) hm[i * mk + j] = (float)(i % 7) - 3.f;
  void *dm, *dverdict;
  CHECK_CUDA(cudaMalloc(&dm, (size_t)(mq * mk) * 4));
  CHECK_CUDA(cudaMalloc(&dverdict, 4));
  CHECK_CUDA(cudaMemcpy(dm, hm, (size_t)(mq * mk) * 4, cudaMemcpyHostToDevice));
  safedit_tensor tm = tensor4(dm, SAFEDIT_F32, 1, 1, mq, mk);
  CHECK_SD(safedit_mask_is_row_constant(&tm, (int32_t *)dverdict, NULL, NULL));
  int32_t verdict = -1;
  CHECK_CUDA(cudaMemcpy(&verdict, dverdict, 4, cudaMemcpyDeviceToHost));
  hm[5 * mk + 17] += 1.f; /* one non-uniform row: kept */
  CHECK_CUDA(cudaMemcpy(dm, hm, (size_t)(mq * mk) * 4, cudaMemcpyHostToDevice));
  CHECK_SD(safedit_mask_is_row_constant(&tm, (int32_t *)dverdict, NULL, NULL));
  int32_t verdict2 = -1;
  CHECK_CUDA(cudaMemcpy(&verdict2, dverdict, 4, cudaMemcpyDeviceToHost));
  printf("mask_is_row_constant: %d then %d\n", verdict, verdict2);
  if (verdict != 1 || verdict2 != 0) return 7;

  /* SW-CFG on [512, 16] f32 */
  const int64_t cn = 512, cf = 16;
  float *hc = malloc((size_t)(cn * cf) * 4), *hu = malloc((size_t)(cn * cf) * 4);
  float *hs = malloc((size_t)cn * 4), *hout = malloc((size_t)(cn * cf) * 4);
  double *c64 = malloc((size_t)(cn * cf) * 8), *u64 = malloc((size_t)(cn * cf) * 8);
  double *s64 = malloc((size_t)cn * 8), *o64 = malloc((size_t)(cn * cf) * 8);
  for (int64_t i = 0; i < cn * cf; ++i) {
    hc[i] = (float)normal01(), hu[i] = (float)normal01();
    c64[i] = hc[i], u64[i] = hu[i];
  }
  for (int64_t i = 0; i < cn; ++i) hs[i] = (float)uniform01(), s64[i] = hs[i];
  void *dc, *du, *ds, *dco;
  CHECK_CUDA(cudaMalloc(&dc, (size_t)(cn * cf) * 4));
  CHECK_CUDA(cudaMalloc(&du, (size_t)(cn * cf) * 4));
  CHECK_CUDA(cudaMalloc(&ds, (size_t)cn * 4));
  CHECK_CUDA(cudaMalloc(&dco, (size_t)(cn * cf) * 4));
  CHECK_CUDA(cudaMemcpy(dc, hc, (size_t)(cn * cf) * 4, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(du, hu, (size_t)(cn * cf) * 4, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(ds, hs, (size_t)cn * 4, cudaMemcpyHostToDevice));
  safedit_tensor tc, tu, tco;
  memset(&tc, 0, sizeof tc);
  tc.dtype = SAFEDIT_F32, tc.ndim = 2, tc.dims[0] = cn, tc.dims[1] = cf, tc.strides[0] = cf,
  tc.strides[1] = 1;
  tu = tc, tco = tc;
  tc.data = dc, tu.data = du, tco.data = dco;
  CHECK_SD(safedit_sw_cfg(&tc, &tu, (const float *)ds, 3.f, 5.f, &tco, NULL));
  CHECK_CUDA(cudaMemcpy(hout, dco, (size_t)(cn * cf) * 4, cudaMemcpyDeviceToHost));
  oracle_sw_cfg(cn, cf, c64, u64, s64, 3.0, 5.0, o64);
  int cfg_ok = 1;
  for (int64_t i = 0; i < cn; ++i)
    for (int64_t j = 0; j < cf; ++j) {
      const int64_t e = i * cf + j;
      const double g = 3.0 + 2.0 * s64[i];
      const double bound = 1e-5 * (fabs(u64[e]) + fabs(g) * fabs(c64[e] - u64[e])) + 1e-30;
      cfg_ok &= fabs((double)hout[e] - o64[e]) <= bound;
    }
  printf("sw_cfg: %s\n", cfg_ok ? "ok" : "MISMATCH");
  if (!cfg_ok) return 8;
  CHECK_SD(safedit_get_device_status(&status, NULL));
  if (status != SAFEDIT_OK) return 9;
  printf("c client ok: %llu library launches\n", (unsigned long long)safedit_kernel_launch_count());
  return 0;
}
