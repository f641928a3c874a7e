"""GPU vs oracle parity of SkipSparse FFN caching (AccelAes summary, B.2):
the tcgen05 projection with fused bias / GELU and scattered output rows, and
the whole block gather -> W1 (+b1, GELU) -> W2 (+b2) -> scatter into the
FFN cache.

Tolerances, from the arithmetic (inputs exactly representable in bf16):
  * one projection without activation: fp32 accumulation over K, one bf16
    rounding of the output (relative <= 2^-9); per element
    |out - ref| <= 2^-8 |ref| + 2^-12 sum_k |a_rk w_nk|  (the second term is
    far above fp32 accumulation error, far below a dropped or doubled k-block);
  * with GELU, and the whole block: the hidden layer is rounded to bf16 and
    GELU's tanh is the hardware approximation (relative error about 2^-11), so
    the comparison is relative Frobenius <= 5e-3 and max |error| <= 2e-2 on
    outputs of unit scale (the attention tolerance);
  * rows that are not recomputed: bit-exact (the cache is untouched).
"""
import numpy as np
import pytest
import torch

import oracle
from spatially_adaptive_dit_b200 import workloads as wl
from tests.gpu_util import ATTN_MAX_ABS, ATTN_REL_FRO, expect_status, f64, rel_fro, sd

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _rand_idx(n_total, k, seed):
    return torch.sort(torch.randperm(n_total, generator=_gen(seed))[:k]).values.to(torch.int32)


def _linear_inputs(M, K, N, seed, B=None):
    g = _gen(seed)
    shape = (M, K) if B is None else (B, M, K)
    a = torch.randn(shape, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    b = 0.1 * torch.randn(N, generator=g)
    return a, w, b


def _check_plain(out, a, w, b):
    """Element-wise bound of a projection without activation (module docstring)."""
    ref = oracle.linear_act(a, w, b, act=0)
    mag = np.abs(f64(a)) @ np.abs(f64(w)).T
    err = np.abs(f64(out) - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -12 * mag
    assert (err <= bound).all(), f"worst excess {float((err - bound).max()):.3e}"


def _check_close(out, ref, what):
    out = np.asarray(out, dtype=np.float64)
    rf = rel_fro(out, ref)
    mx = float(np.abs(out - ref).max()) if out.size else 0.0
    assert rf <= ATTN_REL_FRO and mx <= ATTN_MAX_ABS, f"{what}: relFro={rf:.3e} maxabs={mx:.3e}"


@pytest.mark.parametrize("M,K,N", [(300, 200, 520),     # CTA pairs: ragged rows, k-block and column tails
                                   (128, 64, 256),      # single CTA, exactly one tile
                                   (255, 64, 264),      # single CTA, largest M below the pair tiles
                                   (256, 8, 8),         # CTA pair, one tile, W half of the pair empty
                                   (2560, 512, 2048),   # CTA pairs: 80 tiles, pairs loop, accumulators cycle
                                   (1, 8, 8)])          # smallest legal shape
@pytest.mark.parametrize("bias", [True, False])
def test_projection_plain(M, K, N, bias):
    a, w, b = _linear_inputs(M, K, N, M + K + N)
    b = b if bias else None
    out = torch.full((M, N), 7.0, dtype=torch.bfloat16, device=DEV)
    sd().safedit_gemm_bias_act(a.to(DEV), w.to(DEV), None if b is None else b.to(DEV), 0, None, out)
    expect_status(0)
    _check_plain(out, a, w, b)


@pytest.mark.parametrize("M,K,N", [(300, 200, 520), (2560, 512, 2048)])
def test_projection_gelu(M, K, N):
    a, w, b = _linear_inputs(M, K, N, 3 * M + K)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    sd().safedit_gemm_bias_act(a.to(DEV), w.to(DEV), b.to(DEV), 1, None, out)
    expect_status(0)
    _check_close(f64(out), oracle.linear_act(a, w, b, act=1), "gelu projection")


@pytest.mark.parametrize("M,M_out", [(77, 150),     # single-CTA tiles (M < 256)
                                     (300, 700)])   # CTA-pair tiles with a ragged second row tile
def test_projection_batched_scattered_rows(M, M_out):
    """[B, M, K] input, rows scattered by a shared index into [B, M_out, N];
    rows no index points at keep their bytes."""
    B, K, N = 2, 136, 264
    a, w, b = _linear_inputs(M, K, N, 11, B=B)
    idx = torch.randperm(M_out, generator=_gen(12))[:M].to(torch.int32)  # unique, unsorted
    init = torch.randn(B, M_out, N, generator=_gen(13)).to(torch.bfloat16)
    out = init.to(DEV)
    sd().safedit_gemm_bias_act(a.to(DEV), w.to(DEV), b.to(DEV), 0, idx.to(DEV), out)
    expect_status(0)
    got = out.cpu()
    hit = np.zeros(M_out, dtype=bool)
    hit[idx.numpy()] = True
    for bb in range(B):
        _check_plain(got[bb, idx.long()], a[bb], w, b)
        assert torch.equal(got[bb, torch.from_numpy(~hit)].view(torch.int16),
                           init[bb, torch.from_numpy(~hit)].view(torch.int16))


def test_projection_strided_views():
    """Row strides wider than the row (views into bigger buffers)."""
    M, K, N = 200, 128, 256
    a, w, b = _linear_inputs(M, K, N, 21)
    abig = torch.zeros(M, K + 64, dtype=torch.bfloat16, device=DEV)
    abig[:, 8:8 + K] = a.to(DEV)
    obig = torch.zeros(M, N + 16, dtype=torch.bfloat16, device=DEV)
    sd().safedit_gemm_bias_act(abig[:, 8:8 + K], w.to(DEV), b.to(DEV), 0, None, obig[:, :N])
    expect_status(0)
    _check_plain(obig[:, :N], a, w, b)
    assert not obig[:, N:].any()


def _ffn_block(x, idx, w1, b1, w2, b2, y_cache):
    """The cached FFN on the GPU: gather the focus rows, W1 (+b1, GELU), W2
    (+b2) with the rows scattered back into the cache.  x, y_cache [B,N,D]."""
    B, N, D = x.shape
    k = idx.numel()
    xs = torch.empty(B, 1, k, D, dtype=torch.bfloat16, device=DEV)
    sd().safedit_gather_rows([x.view(B, 1, N, D)], [xs], idx, k)
    h = torch.empty(B, k, w1.shape[0], dtype=torch.bfloat16, device=DEV)
    sd().safedit_gemm_bias_act(xs.view(B, k, D), w1, b1, 1, None, h)
    sd().safedit_gemm_bias_act(h, w2, b2, 0, idx, y_cache)


def test_ffn_block_vs_oracle():
    w = wl.TINY
    B, N, D, F, k = 2, 333, 200, 520, 100
    w1, b1, w2, b2 = wl.ffn_weights(w, D=D, F=F)
    g = _gen(31)
    x = torch.randn(B, N, D, generator=g).to(torch.bfloat16)
    cache = torch.randn(B, N, D, generator=g).to(torch.bfloat16)
    idx = _rand_idx(N, k, 32)
    y = cache.to(DEV)
    _ffn_block(x.to(DEV), idx.to(DEV), w1.to(DEV), b1.to(DEV), w2.to(DEV), b2.to(DEV), y)
    expect_status(0)
    got = y.cpu()
    keep = np.setdiff1d(np.arange(N), idx.numpy())
    for bb in range(B):
        ref = oracle.ffn_cached(x[bb], idx, w1, b1, w2, b2, cache[bb], act=1)
        _check_close(f64(got[bb])[idx.numpy()], ref[idx.numpy()], f"batch {bb}")
        assert torch.equal(got[bb, keep].view(torch.int16), cache[bb, keep].view(torch.int16))


def test_ffn_block_full_size_sampled():
    """The 2560^2 workload's FFN (B=2, N=25600, D=2304, F=9216, |S|=7680) in
    the launch configuration the benchmark times; sampled focus rows against
    the oracle, sampled background rows bit-exact."""
    w = wl.W2560
    B, N, D, F, k = w.B, w.N, w.D_model, w.D_ff, w.k
    w1, b1, w2, b2 = wl.ffn_weights(w)
    x, cache = wl.ffn_states(w)
    idx = _rand_idx(N, k, 41)
    y = cache.to(DEV)
    _ffn_block(x.to(DEV), idx.to(DEV), w1.to(DEV), b1.to(DEV), w2.to(DEV), b2.to(DEV), y)
    expect_status(0)
    picks = torch.cat([torch.tensor([0, k - 1]), torch.randperm(k, generator=_gen(42))[:14]])
    rows = idx[picks].long()
    keep = torch.from_numpy(np.setdiff1d(np.arange(N), idx.numpy()))
    keep = keep[torch.randperm(keep.numel(), generator=_gen(43))[:64]]
    for bb in range(B):
        ref = oracle.ffn_cached(x[bb, rows], None, w1, b1, w2, b2, np.zeros((len(rows), D)), act=1)
        _check_close(f64(y[bb, rows.to(DEV)]), ref, f"batch {bb}")
        assert torch.equal(y[bb, keep.to(DEV)].cpu().view(torch.int16), cache[bb, keep].view(torch.int16))


def test_projection_argument_and_device_errors():
    a, w, b = _linear_inputs(64, 64, 64, 51)
    a, w, b = a.to(DEV), w.to(DEV), b.to(DEV)
    out = torch.empty(64, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(sd().SafeditError) as e:
        sd().safedit_gemm_bias_act(a, w[:60], b, 0, None, out[:, :60])  # N % 8 != 0
    assert e.value.code == sd().ERR_ALIGNMENT
    with pytest.raises(sd().SafeditError) as e:
        sd().safedit_gemm_bias_act(a.float(), w, b, 0, None, out)
    assert e.value.code == sd().ERR_DTYPE
    with pytest.raises(sd().SafeditError) as e:
        sd().safedit_gemm_bias_act(a, w, b, 2, None, out)
    assert e.value.code == sd().ERR_INVALID_ARG
    with pytest.raises(sd().SafeditError) as e:
        sd().safedit_gemm_bias_act(a, w[:, :32], b, 0, None, out)
    assert e.value.code == sd().ERR_SHAPE
    n0 = sd().safedit_kernel_launch_count()
    sd().safedit_gemm_bias_act(a[:0], w, b, 0, None, out[:0])  # M == 0: no launch
    assert sd().safedit_kernel_launch_count() == n0
    # an index outside the output: flagged on the device, that row skipped
    idx = torch.arange(64, dtype=torch.int32, device=DEV)
    idx[5] = 64
    out.zero_()
    sd().safedit_gemm_bias_act(a, w, b, 0, idx, out)
    expect_status(sd().ERR_INDEX)
    ref = torch.empty_like(out)
    sd().safedit_gemm_bias_act(a, w, b, 0, None, ref)
    expect_status(0)
    rows = torch.tensor([r for r in range(64) if r != 5], device=DEV)
    assert torch.equal(out[rows], ref[rows])


def test_gathered_qkv_projection_feeds_srsu():
    """SkipSparse on one attention layer: only the focus rows are projected
    (x_S W_qkv^T + b, fused q|k|v output with heads inner), their K/V replace
    the cached rows of the state, and their Q attends over the whole state,
    read through strided views of the projection output.  Against the oracle
    composed from gather, linear_act, scatter and attn_subset in fp64.
    Tolerance: two bf16 roundings in sequence (projection outputs, then the
    attention's P and O), each about 2e-3 relative: relative Frobenius <= 1e-2."""
    B, H, d, N, k = 2, 2, 64, 384, 100
    D = H * d
    g = _gen(61)
    x = torch.randn(B, N, D, generator=g).to(torch.bfloat16)
    wqkv = (torch.randn(3 * D, D, generator=g) / D ** 0.5).to(torch.bfloat16)
    bqkv = 0.02 * torch.randn(3 * D, generator=g)
    k_state = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v_state = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    idx = _rand_idx(N, k, 62)
    # GPU: gather -> projection -> scatter K/V -> compact-query attention
    d_idx = idx.to(DEV)
    xs = torch.empty(B, 1, k, D, dtype=torch.bfloat16, device=DEV)
    sd().safedit_gather_rows([x.to(DEV).view(B, 1, N, D)], [xs], d_idx, k)
    qkv = torch.empty(B, k, 3 * D, dtype=torch.bfloat16, device=DEV)
    sd().safedit_gemm_bias_act(xs.view(B, k, D), wqkv.to(DEV), bqkv.to(DEV), 0, None, qkv)
    q_s, k_s, v_s = (qkv.view(B, k, 3, H, d)[:, :, j].permute(0, 2, 1, 3) for j in range(3))
    ks_d, vs_d = k_state.to(DEV), v_state.to(DEV)
    sd().safedit_scatter_state([k_s, v_s], [ks_d, vs_d], d_idx, k)
    out = torch.empty(B, H, k, d, dtype=torch.bfloat16, device=DEV)
    sd().safedit_attn_subset(q_s, ks_d, vs_d, None, 0, None, None, 0.0, out, 0)
    expect_status(0)
    # oracle composition
    for bb in range(B):
        x_s = oracle.gather_rows(x[bb].view(torch.int16).numpy(), idx)
        x_s = torch.from_numpy(x_s).view(torch.bfloat16)
        proj = oracle.linear_act(x_s, wqkv, bqkv, act=0).reshape(k, 3, H, d)
        for h in range(H):
            kst = oracle.scatter_rows(proj[:, 1, h], f64(k_state[bb, h]), idx)
            vst = oracle.scatter_rows(proj[:, 2, h], f64(v_state[bb, h]), idx)
            ref = oracle.attn_subset(proj[:, 0, h], kst, vst)
            rf = rel_fro(f64(out[bb, h]), ref)
            assert rf <= 1e-2, f"b{bb}h{h}: relFro={rf:.3e}"


def test_w2_projection_at_bench_shape_scattered_into_cache():
    """The FFN W2 projection of the 2560^2 workload exactly as the benchmark
    launches it: the bf16 hidden layer of every focus row (B = 2 batches of
    |S| = 7680 rows, K = 4D = 9216, N = D = 2304, so 144 k-blocks per tile)
    times W2 plus b2, each row written to its token's row of the FFN cache
    (CTA-pair kernel).  Sampled rows of both batches against the oracle with
    the per-element bound of a projection; the rows no focus token maps to
    keep their bytes."""
    w = wl.W2560
    B, k, D, F = w.B, w.k, w.D_model, w.D_ff
    w1, b1, w2, b2 = wl.ffn_weights(w)
    score = wl.blob_scores(wl.Workload("2560b", 2, B=1, H=1, N=w.N, d=w.d, L=1, n_valid=1,
                                       rho=w.rho, grid=w.grid)).to(DEV)
    idx = torch.empty(k, dtype=torch.int32, device=DEV)
    sd().safedit_partition_finalize(score, w.N, k, idx, None, None)
    hid = wl.normal((B, k, F), w, 777, device=DEV)      # a bf16 hidden layer of unit scale
    y0 = wl.ffn_states(w)[1]                            # the FFN cache [B, N, D] bf16
    y = y0.to(DEV)
    sd().safedit_gemm_bias_act(hid, w2.to(DEV), b2.to(DEV), 0, idx, y)
    expect_status(0)
    ic = idx.cpu().long()
    rows = np.linspace(0, k - 1, 40).astype(np.int64)
    for bb in range(B):
        got = y[bb, ic[rows].to(DEV)].cpu()
        _check_plain(got, hid[bb, torch.as_tensor(rows, device=DEV)].cpu(), w2, b2)
    hit = torch.zeros(w.N, dtype=torch.bool)
    hit[ic] = True
    keep = torch.nonzero(~hit).flatten()[::97]
    assert torch.equal(y[:, keep.to(DEV)].cpu().view(torch.int16), y0[:, keep].view(torch.int16))
