"""GPU vs oracle parity of the bandwidth kernels: state scatter / gather,
SW-CFG, PCSP score aggregation and split, and the mask-elision check."""
import os

import numpy as np
import pytest
import torch

import oracle
from spatially_adaptive_dit_b200 import workloads as wl
from tests.gpu_util import CFG_REL, expect_status, sd

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _rand_idx(n_total, k, seed):
    g = _gen(seed)
    return torch.sort(torch.randperm(n_total, generator=g)[:k]).values.to(torch.int32)


# ----------------------------------------------------------- scatter / gather
@pytest.mark.parametrize("D,dtype,B,H,N,k", [(96, torch.bfloat16, 2, 3, 1000, 300),
                                              (64, torch.bfloat16, 1, 2, 256, 64),
                                              (128, torch.bfloat16, 1, 4, 517, 517),
                                              (16, torch.float32, 2, 2, 333, 1),
                                              (2304, torch.bfloat16, 2, 1, 700, 300),  # rows wider than a block
                                              (1100, torch.float32, 1, 2, 90, 45)])
def test_scatter_gather_bit_exact(D, dtype, B, H, N, k):
    g = _gen(D + N)
    idx = _rand_idx(N, k, N + k)
    srcs = [torch.randn(B, H, k, D, generator=g).to(dtype) for _ in range(3)]
    dsts = [torch.randn(B, H, N, D, generator=g).to(dtype) for _ in range(3)]
    d_src = [s.to(DEV) for s in srcs]
    d_dst = [d.to(DEV) for d in dsts]
    d_idx = idx.to(DEV)
    sd().safedit_scatter_state(d_src, d_dst, d_idx, k)
    expect_status(0)
    itype = torch.int16 if dtype == torch.bfloat16 else torch.int32
    for s, d, dd in zip(srcs, dsts, d_dst):
        for b in range(B):
            for h in range(H):
                ref = oracle.scatter_rows(s[b, h].view(itype).numpy(), d[b, h].view(itype).numpy(), idx)
                assert np.array_equal(dd[b, h].cpu().view(itype).numpy(), ref)
    # gather back the S rows
    outs = [torch.empty(B, H, k, D, dtype=dtype, device=DEV) for _ in range(3)]
    sd().safedit_gather_rows(d_dst, outs, d_idx, k)
    expect_status(0)
    for s, o in zip(srcs, outs):
        assert torch.equal(o.cpu().view(itype), s.view(itype))


def test_scatter_strided_views_and_oob_index():
    B, H, N, D, k = 2, 2, 64, 64, 10
    base = torch.zeros(B, N, H, D, dtype=torch.bfloat16, device=DEV)  # [B,N,H,D] storage
    dst = base.permute(0, 2, 1, 3)                                     # strided [B,H,N,D] view
    src = torch.randn(B, H, k, D, device=DEV).to(torch.bfloat16)
    idx = torch.arange(0, 2 * k, 2, dtype=torch.int32, device=DEV)
    sd().safedit_scatter_state([src], [dst], idx, k)
    expect_status(0)
    assert torch.equal(dst[:, :, idx.long()], src)
    bad = idx.clone()
    bad[3] = N + 5
    sd().safedit_scatter_state([src], [dst], bad, k)
    expect_status(sd().ERR_INDEX)


# -------------------------------------------------------------------- SW-CFG
@pytest.mark.parametrize("N,F", [(4096, 16), (25600, 16), (1000, 13), (257, 4096)])
def test_sw_cfg(N, F):
    g = _gen(N * 7 + F)
    c = torch.randn(N, F, generator=g)
    u = torch.randn(N, F, generator=g)
    s = torch.rand(N, generator=g)
    s[:3] = torch.tensor([0.0, 1.0, 0.5])
    out = torch.empty(N, F, device=DEV)
    sd().safedit_sw_cfg(c.to(DEV), u.to(DEV), s.to(DEV), 3.0, 5.0, out)
    expect_status(0)
    ref = oracle.sw_cfg(c, u, s, 3.0, 5.0)
    gam = 3.0 + 2.0 * s.double().numpy()[:, None]
    scale = np.abs(u.double().numpy()) + np.abs(gam) * np.abs((c.double() - u.double()).numpy())
    err = np.abs(out.cpu().double().numpy() - ref)
    assert np.all(err <= CFG_REL * scale + 1e-30)
    # in-place (out aliases eps_c) and plain CFG (gamma_ctx == gamma_sens)
    cd = c.to(DEV)
    sd().safedit_sw_cfg(cd, u.to(DEV), s.to(DEV), 4.0, 4.0, cd)
    expect_status(0)
    ref2 = oracle.sw_cfg(c, u, s, 4.0, 4.0)
    assert np.abs(cd.cpu().double().numpy() - ref2).max() <= 1e-5 * (1 + np.abs(ref2).max())


@pytest.mark.parametrize("N,F,vec", [(4096, 16, True), (300, 6, False), (257, 16, False)])
def test_sw_cfg_bf16_predictions(N, F, vec):
    """bf16 eps_c / eps_u (widened exactly), f32 output; vector path (F % 4
    == 0, 8-byte aligned rows) and the scalar path (odd widths, and a view
    whose rows start off the 8-byte boundary)."""
    g = _gen(N + 13 * F)
    c = torch.randn(N, F, generator=g).to(torch.bfloat16)
    u = torch.randn(N, F, generator=g).to(torch.bfloat16)
    s = torch.rand(N, generator=g)
    cd, ud = c.to(DEV), u.to(DEV)
    if not vec and F % 4 == 0:  # same values at an address 2 bytes past an 8-byte boundary
        cb = torch.empty(N * F + 1, dtype=torch.bfloat16, device=DEV)
        cb[1:].copy_(cd.flatten())
        cd = cb[1:].view(N, F)
    out = torch.empty(N, F, device=DEV)
    sd().safedit_sw_cfg(cd, ud, s.to(DEV), 3.0, 5.0, out)
    expect_status(0)
    ref = oracle.sw_cfg(c.double(), u.double(), s, 3.0, 5.0)
    gam = 3.0 + 2.0 * s.double().numpy()[:, None]
    scale = np.abs(u.double().numpy()) + np.abs(gam) * np.abs((c.double() - u.double()).numpy())
    err = np.abs(out.cpu().double().numpy() - ref)
    assert np.all(err <= CFG_REL * scale + 1e-30)
    with pytest.raises(sd().SafeditError) as e:  # mixed input types
        sd().safedit_sw_cfg(cd, u.float().to(DEV), s.to(DEV), 3.0, 5.0, out)
    assert e.value.code == sd().ERR_DTYPE


# ------------------------------------------------------------- partition PCSP
@pytest.mark.parametrize("H,N,L,nvalid", [(24, 4096, 256, 128), (2, 256, 32, 20), (3, 1000, 30, 25),
                                          (4, 300, 512, 400)])
def test_partition_accumulate_and_finalize(H, N, L, nvalid):
    g = _gen(H * N + L)
    logits = torch.randn(H, N, L, generator=g)
    logits[:, :, nvalid:] = float("-inf")
    P = torch.softmax(logits, dim=-1).float()  # a probability tensor of the right structure
    content = torch.zeros(L, dtype=torch.uint8)
    content[1:nvalid - 1] = 1
    score = torch.zeros(N, dtype=torch.float64, device=DEV)
    Pd = P.to(DEV)
    sd().safedit_partition_accumulate(Pd, content.to(DEV), score)
    sd().safedit_partition_accumulate(Pd, content.to(DEV), score)  # two warm-up calls
    expect_status(0)
    ref = oracle.partition_accumulate(P, content)
    ref = oracle.partition_accumulate(P, content, ref)
    got = score.cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()
    # split: the GPU and the oracle take the same score array -> bit-exact
    for k in (0, 1, N // 4, wl.k_of(wl.W1024.rho, N), N - 1, N):
        idx_s = torch.empty(max(k, 1), dtype=torch.int32, device=DEV)
        idx_c = torch.empty(max(N - k, 1), dtype=torch.int32, device=DEV)
        s = torch.empty(N, dtype=torch.float32, device=DEV)
        sd().safedit_partition_finalize(score, N, k, idx_s, idx_c, s)
        expect_status(0)
        r_s, r_c, r_sv = oracle.partition_select(got, k)
        assert np.array_equal(idx_s.cpu().numpy()[:k], r_s)
        assert np.array_equal(idx_c.cpu().numpy()[:N - k], r_c)
        assert np.array_equal(s.cpu().numpy(), r_sv)
    # scores from the oracle's own accumulation: exact except near the threshold
    k = wl.k_of(wl.W1024.rho, N)
    r_s, _, _ = oracle.partition_select(ref, k)
    idx_s = torch.empty(k, dtype=torch.int32, device=DEV)
    sd().safedit_partition_finalize(score, N, k, idx_s, None, None)
    tau = np.sort(ref)[::-1][k - 1]
    near = np.abs(ref - tau) <= 1e-6 * abs(tau)
    a = set(idx_s.cpu().numpy().tolist()) - set(np.nonzero(near)[0].tolist())
    b = set(r_s.tolist()) - set(np.nonzero(near)[0].tolist())
    assert a == b


@pytest.mark.parametrize("H,N,L,nvalid", [(24, 4096, 256, 128), (3, 1000, 30, 25), (4, 300, 512, 400),
                                          (2, 700, 1024, 900)])
def test_partition_accumulate_bf16_probabilities(H, N, L, nvalid):
    """P stored in bf16 (vector path when L % 8 == 0, the scalar path at
    L = 30), widened exactly: against the oracle on the same bf16 values."""
    g = _gen(7 * H * N + L)
    logits = torch.randn(H, N, L, generator=g)
    logits[:, :, nvalid:] = float("-inf")
    P = torch.softmax(logits, dim=-1).to(torch.bfloat16)
    content = torch.zeros(L, dtype=torch.uint8)
    content[1:nvalid - 1] = 1
    score = torch.zeros(N, dtype=torch.float64, device=DEV)
    sd().safedit_partition_accumulate(P.to(DEV), content.to(DEV), score)
    expect_status(0)
    ref = oracle.partition_accumulate(P.double(), content)
    assert np.abs(score.cpu().numpy() - ref).max() <= 1e-12 * np.abs(ref).max()
    # a strided view (every other head of a larger tensor) takes the same path
    big = torch.zeros(2 * H, N, L, dtype=torch.bfloat16, device=DEV)
    big[::2] = P.to(DEV)
    score.zero_()
    sd().safedit_partition_accumulate(big[::2], content.to(DEV), score)
    expect_status(0)
    assert np.abs(score.cpu().numpy() - ref).max() <= 1e-12 * np.abs(ref).max()


def test_partition_finalize_ties_and_signed_zero():
    N = 5000
    g = _gen(99)
    score = torch.randint(0, 7, (N,), generator=g).double()
    score[::17] = -0.0
    score[::19] = 0.0
    for k in (1, 17, 2500, 4999):
        d = score.to(DEV)
        idx_s = torch.empty(k, dtype=torch.int32, device=DEV)
        idx_c = torch.empty(N - k, dtype=torch.int32, device=DEV)
        s = torch.empty(N, device=DEV)
        sd().safedit_partition_finalize(d, N, k, idx_s, idx_c, s)
        expect_status(0)
        r_s, r_c, r_sv = oracle.partition_select(score.numpy(), k)
        assert np.array_equal(idx_s.cpu().numpy(), r_s)
        assert np.array_equal(idx_c.cpu().numpy(), r_c)
        assert np.array_equal(s.cpu().numpy(), r_sv)


def test_partition_finalize_blob_scores_stress_config():
    w = wl.STRESS
    score = wl.blob_scores(w)
    k = w.k
    idx_s = torch.empty(k, dtype=torch.int32, device=DEV)
    idx_c = torch.empty(w.N - k, dtype=torch.int32, device=DEV)
    s = torch.empty(w.N, device=DEV)
    sd().safedit_partition_finalize(score.to(DEV), w.N, k, idx_s, idx_c, s)
    expect_status(0)
    r_s, r_c, r_sv = oracle.partition_select(score.numpy(), k)
    assert np.array_equal(idx_s.cpu().numpy(), r_s)
    assert np.array_equal(idx_c.cpu().numpy(), r_c)
    assert np.array_equal(s.cpu().numpy(), r_sv)


# ---------------------------------------------------------------- mask check
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("kind", wl.MASK_KINDS)
def test_mask_kinds_small(kind, dtype):
    w = wl.TINY
    m = wl.mask(w, kind, dtype=dtype)
    v = torch.zeros(1, dtype=torch.int32, device=DEV)
    flags = torch.zeros(m.shape[:-1].numel(), dtype=torch.uint8, device=DEV)
    sd().safedit_mask_is_row_constant(m.to(DEV), v, flags)
    expect_status(0)
    rv, rf = oracle.mask_row_constant(m)
    assert int(v.item()) == rv == (1 if kind in ("zero", "rowconst") else 0)
    assert np.array_equal(flags.cpu().numpy(), rf.reshape(-1))
    v2 = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    sd().safedit_mask_is_row_constant(m.to(DEV), v2, None)  # early-exit path
    expect_status(0)
    assert int(v2.item()) == rv


def test_mask_edge_cases():
    rows = []
    golden = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "mask_rows_hand.txt")
    for ln in open(golden):
        if ln.strip() and not ln.startswith("#"):
            e, vals = ln.split("|")
            rows.append((int(e), [float(x) for x in vals.split()]))
    expect = np.array([e for e, _ in rows], dtype=np.uint8)
    m32 = torch.tensor([r for _, r in rows], dtype=torch.float32)
    for dt in (torch.float32, torch.bfloat16, torch.float16):
        mm = m32.to(dt)
        # pad rows to 8 columns of the row's first value so vector and scalar paths both run
        for cols in (5, 8 * 9):
            full = torch.cat([mm, mm[:, :1].expand(-1, cols - 5)], dim=1) if cols > 5 else mm
            v = torch.zeros(1, dtype=torch.int32, device=DEV)
            fl = torch.zeros(full.shape[0], dtype=torch.uint8, device=DEV)
            sd().safedit_mask_is_row_constant(full.to(DEV), v, fl)
            expect_status(0)
            rv, rf = oracle.mask_row_constant(full)
            assert np.array_equal(fl.cpu().numpy(), rf) and int(v.item()) == rv
            if cols == 5 and dt == torch.float32:  # the hand verdicts are for fp32 values
                assert np.array_equal(rf, expect)
    # bool masks, 4-D, with a broadcast head dim (stride 0) and a broadcast query dim
    bm = torch.ones(2, 1, 64, 96, dtype=torch.bool)
    bm[1, 0, 5, 90] = False
    v = torch.zeros(1, dtype=torch.int32, device=DEV)
    fl = torch.zeros(2 * 3 * 64, dtype=torch.uint8, device=DEV)
    sd().safedit_mask_is_row_constant(bm.to(DEV).expand(2, 3, 64, 96), v, fl)
    expect_status(0)
    rv, rf = oracle.mask_row_constant(bm.expand(2, 3, 64, 96).contiguous())
    assert int(v.item()) == rv == 0 and np.array_equal(fl.cpu().numpy(), rf.reshape(-1))
    kp = torch.zeros(2, 1, 1, 1000, dtype=torch.bfloat16, device=DEV)  # key-padding style, all valid
    sd().safedit_mask_is_row_constant(kp.expand(2, 1, 4096, 1000), v, None)
    expect_status(0)
    assert int(v.item()) == 1


@pytest.mark.slow
def test_mask_stress_config_full_size():
    """[1,1,16384,16384] bf16 masks of the four kinds; verdict and sampled row flags."""
    w = wl.STRESS
    rows = np.linspace(0, w.N - 1, 97).astype(np.int64)
    for kind in wl.MASK_KINDS:
        m = wl.mask(w, kind, device=DEV)
        v = torch.zeros(1, dtype=torch.int32, device=DEV)
        fl = torch.zeros(w.N, dtype=torch.uint8, device=DEV)
        sd().safedit_mask_is_row_constant(m, v, fl)
        expect_status(0)
        rv, rf = oracle.mask_row_constant(m[0, 0, torch.as_tensor(rows, device=DEV)].cpu())
        assert np.array_equal(fl.cpu().numpy()[rows], rf)
        assert int(v.item()) == (1 if kind in ("zero", "rowconst") else 0)
        del m


# ----------------------------------------------------------------- StepCache
@pytest.mark.parametrize("N,F,w", [(4096, 16, 0.5), (25600, 16, 1.0), (1000, 13, -0.25), (257, 4096, 2.0)])
def test_stepcache_sw_cfg(N, F, w):
    g = _gen(N * 3 + F)
    ca, cb, ua, ub = (torch.randn(N, F, generator=g) for _ in range(4))
    s = torch.rand(N, generator=g)
    out = torch.empty(N, F, device=DEV)
    sd().safedit_stepcache_sw_cfg(ca.to(DEV), cb.to(DEV), ua.to(DEV), ub.to(DEV), s.to(DEV), w, 3.0, 5.0, out)
    expect_status(0)
    ref = oracle.stepcache_sw_cfg(ca, cb, ua, ub, s, w, 3.0, 5.0)
    gam = (3.0 + 2.0 * s.double().numpy())[:, None]
    mag = (1 + abs(w)) * (ca.abs() + cb.abs() + ua.abs() + ub.abs()).double().numpy()
    err = np.abs(out.cpu().double().numpy() - ref)
    assert np.all(err <= CFG_REL * (1 + gam) * mag + 1e-30)


def test_stepcache_sw_cfg_large_sampled():
    """A bandwidth-sized call (grid-stride loop over many passes): sampled rows
    against the oracle, every row against the same combine in fp32 torch on the
    device being finite and unchanged where the branches agree."""
    N, F, w = 25600, 4096, 0.5
    g = torch.Generator(device=DEV).manual_seed(77)
    ca, cb, ua, ub = (torch.randn(N, F, generator=g, device=DEV) for _ in range(4))
    s = torch.rand(N, generator=g, device=DEV)
    out = torch.full((N, F), float("nan"), device=DEV)
    sd().safedit_stepcache_sw_cfg(ca, cb, ua, ub, s, w, 3.0, 5.0, out)
    expect_status(0)
    assert bool(torch.isfinite(out).all())  # every element was written
    rows = torch.cat([torch.tensor([0, N - 1]), torch.randperm(N, generator=_gen(78))[:62]]).to(DEV)
    sub = [t[rows].cpu() for t in (ca, cb, ua, ub)]
    ref = oracle.stepcache_sw_cfg(*sub, s[rows].cpu(), w, 3.0, 5.0)
    gam = (3.0 + 2.0 * s[rows].cpu().double().numpy())[:, None]
    mag = (1 + abs(w)) * sum(t.abs() for t in sub).double().numpy()
    err = np.abs(out[rows].cpu().double().numpy() - ref)
    assert np.all(err <= CFG_REL * (1 + gam) * mag + 1e-30)


@pytest.mark.parametrize("n", [1, 3, 1000, 1024, 1025, 36864])
def test_partition_finalize_sizes_and_degenerate_scores(n):
    """Sizes below, at and above one token per thread (the compaction gives
    each of the 1024 threads a contiguous run of tokens) and the 3072^2 token
    count; all-equal scores (every token ties: the lowest indices win,
    s = 0) and scores in a few distinct values.  (The oracle's selection is
    quadratic: the large size takes one k.)"""
    g = _gen(n + 5)
    for kind in ("random", "equal", "few"):
        if kind == "random":
            score = torch.randn(n, generator=g, dtype=torch.float64)
        elif kind == "equal":
            score = torch.full((n,), 0.25, dtype=torch.float64)
        else:
            score = torch.randint(-3, 4, (n,), generator=g).double() * 0.5
        for k in (sorted({0, 1, n // 3, n - 1, n}) if n <= 1025 else [n // 3]):
            idx_s = torch.full((max(k, 1),), -7, dtype=torch.int32, device=DEV)
            idx_c = torch.full((max(n - k, 1),), -7, dtype=torch.int32, device=DEV)
            s = torch.empty(n, device=DEV)
            sd().safedit_partition_finalize(score.to(DEV), n, k, idx_s, idx_c, s)
            expect_status(0)
            r_s, r_c, r_sv = oracle.partition_select(score.numpy(), k)
            assert np.array_equal(idx_s.cpu().numpy()[:k], r_s), (kind, k)
            assert np.array_equal(idx_c.cpu().numpy()[:n - k], r_c), (kind, k)
            assert np.array_equal(s.cpu().numpy(), r_sv), (kind, k)


def test_partition_finalize_nan_score_is_reported():
    score = torch.randn(5000, dtype=torch.float64)
    score[1234] = float("nan")
    idx_s = torch.empty(100, dtype=torch.int32, device=DEV)
    sd().safedit_partition_finalize(score.to(DEV), 5000, 100, idx_s, None, None)
    expect_status(sd().ERR_INVALID_ARG)
