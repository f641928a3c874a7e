"""GPU vs oracle parity of the SRSU subset attention / CAR dense anchor kernel
(tcgen05/TMEM), from tiny ragged cases to the full-size launch configuration
the benchmark times (sampled rows), plus the kernel's edge cases."""
import numpy as np
import pytest
import torch

import oracle
from spatially_adaptive_dit_b200 import workloads as wl
from tests.gpu_util import check_attn, expect_status, f64, sd

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF = torch.bfloat16


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _rand_idx(n_total, k, seed):
    return torch.sort(torch.randperm(n_total, generator=_gen(seed))[:k]).values.to(torch.int32)


def _qkv(B, H, Nq, Nk, D, seed):
    g = _gen(seed)
    q = torch.randn(B, H, Nq, D, generator=g).to(BF)
    k = torch.randn(B, H, Nk, D, generator=g).to(BF)
    v = torch.randn(B, H, Nk, D, generator=g).to(BF)
    return q, k, v


def run(q, k, v, idx=None, pad=None, bias=None, scale=0.0, out=None, scattered=False, status=0):
    B, H, Nq, D = q.shape
    n = Nq if idx is None else idx.numel()
    if out is None:
        out = torch.zeros(B, H, Nq if scattered else n, D, dtype=BF, device=DEV)
    sd().safedit_attn_subset(q, k, v, idx, n, pad, bias, scale, out, int(scattered))
    expect_status(status)
    return out


def oracle_rows(q, k, v, idx, b, h, rows=None, pad=None, bias=None, scale=None):
    """Oracle output rows r (positions in idx) of slice (b,h)."""
    qi = q[b, h]
    sel = np.arange(len(idx)) if rows is None else np.asarray(rows)
    ix = np.asarray(idx)[sel].astype(np.int32)
    brow = None
    if bias is not None:
        bb = bias[b, 0 if bias.shape[1] == 1 else h]
        brow = f64(bb[torch.as_tensor(ix, dtype=torch.long, device=bb.device)])
    return oracle.attn_subset(f64(qi), f64(k[b, h]), f64(v[b, h]), ix,
                              pad=None if pad is None else f64(pad[b]), bias_rows=brow, scale=scale)


@pytest.mark.parametrize("B,H,Nq,Nk,D,k_rows", [(1, 2, 256, 256, 64, 64),     # tiny config shape
                                                 (2, 3, 300, 300, 96, 77),     # ragged rows and keys
                                                 (1, 2, 517, 200, 128, 130),   # ragged, d=128
                                                 (1, 1, 64, 1, 96, 3),         # one key
                                                 (1, 2, 2000, 700, 96, 600)])  # several tiles, 3 CTAs
def test_subset_matches_oracle(B, H, Nq, Nk, D, k_rows):
    q, k, v = _qkv(B, H, Nq, Nk, D, seed=B * 1000 + Nq + D)
    idx = _rand_idx(Nq, k_rows, seed=Nk + k_rows)
    qd, kd, vd, idd = q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV)
    out = run(qd, kd, vd, idd)
    for b in range(B):
        for h in range(H):
            ref = oracle_rows(q, k, v, idx.numpy(), b, h)
            check_attn(f64(out[b, h]), ref, f"b{b}h{h}")


@pytest.mark.parametrize("N,D", [(256, 64), (129, 96), (384, 128)])
def test_dense_anchor_and_subset_rows_agree(N, D):
    """idx = NULL is the CAR anchor: all rows.  An SRSU row must equal the
    same row of the anchor (the S queries attend to the global K/V)."""
    q, k, v = _qkv(1, 2, N, N, D, seed=N + D)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    dense = run(qd, kd, vd)
    for h in range(2):
        ref = oracle.attn_dense(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]))
        check_attn(f64(dense[0, h]), ref, f"dense h{h}")
    idx = _rand_idx(N, N // 3, seed=5)
    sub = run(qd, kd, vd, idx.to(DEV))
    assert torch.equal(sub, dense[:, :, idx.long()])


def test_scattered_output_leaves_context_rows_untouched():
    B, H, N, D, kr = 2, 2, 700, 96, 211
    q, k, v = _qkv(B, H, N, N, D, seed=77)
    idx = _rand_idx(N, kr, seed=78)
    state = torch.randn(B, H, N, D, generator=_gen(79)).to(BF)
    st_d = state.to(DEV)
    run(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), out=st_d, scattered=True)
    mask = torch.ones(N, dtype=torch.bool)
    mask[idx.long()] = False
    assert torch.equal(st_d.cpu()[:, :, mask], state[:, :, mask])
    for b in range(B):
        for h in range(H):
            ref = oracle_rows(q, k, v, idx.numpy(), b, h)
            check_attn(f64(st_d[b, h, idx.long()]), ref)


def test_kept_masks_key_padding_and_bias():
    """Kept semantic masks: key padding (exact zero weight) and a non-uniform
    bias, in f32 and bf16, with a per-head and a broadcast head dim."""
    B, H, N, D, kr = 2, 2, 640, 128, 150
    q, k, v = _qkv(B, H, N, N, D, seed=11)
    idx = _rand_idx(N, kr, seed=12)
    pad = torch.zeros(B, N)
    pad[0, N - N // 8:] = float("-inf")
    pad[1, ::3] = float("-inf")
    g = _gen(13)
    for bias in (torch.randn(B, H, N, N, generator=g), torch.randn(B, 1, N, N, generator=g).to(BF)):
        bd = bias.to(DEV)
        out = run(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), pad=pad.to(DEV), bias=bd)
        for b in range(B):
            for h in range(H):
                ref = oracle_rows(q, k, v, idx.numpy(), b, h, pad=pad, bias=bias)
                check_attn(f64(out[b, h]), ref, f"b{b}h{h}")
    # padded keys carry no weight: garbage in their values must not leak
    vg = v.clone()
    vg[0, :, N - N // 8:] = 1e4
    o1 = run(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), pad=pad.to(DEV))
    o2 = run(q.to(DEV), k.to(DEV), vg.to(DEV), idx.to(DEV), pad=pad.to(DEV))
    assert torch.equal(o1[0], o2[0])


@pytest.mark.parametrize("D", [64, 96, 128])
@pytest.mark.parametrize("kind", ["pad", "bias_f32", "bias_bf16", "pad+bias_f32", "pad+bias_bf16"])
def test_kept_mask_variants_ragged_tail_and_max_jumps(D, kind):
    """Every kept-mask kernel variant.  The last key tile is ragged, ending
    inside the first and inside the second 64-column pass; the additive terms
    raise the running max by far more than the lazy-rescale threshold inside
    every pass position of a tile (the earlier passes' probabilities, already
    in TMEM, are then rescaled); padded keys hold garbage values that must get
    exactly zero weight."""
    B, H, kr = 1, 2, 150
    for N in (696, 600):  # last tile: 56 keys, 88 keys
        q, k, v = _qkv(B, H, N, N, D, seed=1000 + N + D)
        idx = _rand_idx(N, kr, seed=1001 + N)
        pad = bias = None
        if kind.startswith("pad"):
            pad = torch.zeros(B, N)
            pad[:, 5::7] = float("-inf")
            pad[:, 128 + 10:128 + 20] += 9.0        # tile 1, first pass
            pad[:, 256 + 70:256 + 90] += 18.0       # tile 2, second pass
        if "bias" in kind:
            g = _gen(1002 + N)
            bias = torch.randn(B, H if kind.endswith("f32") else 1, N, N, generator=g) * 0.5
            bias[..., ::2, 384 + 64:384 + 80] += 12.0   # tile 3, second pass, even query rows
            bias[..., 1::2, 512 + 3:512 + 9] += 10.0    # ragged tile 4, first pass, odd rows
            # with an f32 bias the passes are 32 keys wide: jumps in the second
            # and in the fourth pass of tile 2 as well
            bias[..., 1::3, 256 + 40:256 + 44] += 14.0
            bias[..., 2::3, 256 + 100:256 + 110] += 16.0
            if kind.endswith("bf16"):
                bias = bias.to(BF)
        dv = lambda t: None if t is None else t.to(DEV)
        out = run(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), pad=dv(pad), bias=dv(bias))
        for h in range(H):
            ref = oracle_rows(q, k, v, idx.numpy(), 0, h, pad=pad, bias=bias)
            check_attn(f64(out[0, h]), ref, f"{kind} D={D} N={N} h{h}")
        if pad is not None:
            vg = v.clone()
            vg[:, :, 5::7] = 1e4
            o2 = run(q.to(DEV), k.to(DEV), vg.to(DEV), idx.to(DEV), pad=dv(pad), bias=dv(bias))
            assert torch.equal(out, o2)


@pytest.mark.parametrize("D", [96, 128])
@pytest.mark.parametrize("bias_kind", [None, "bf16", "f32"])
def test_key_tiles_of_padding_are_skipped_exactly(D, bias_kind):
    """Key tiles whose pad is -inf throughout carry exactly zero weight and are
    skipped: dead tiles first, in the middle and last (the ragged one), with
    live tiles between them; garbage in the dead tiles' values must not leak,
    and the result must match the oracle."""
    B, H, N, kr = 1, 2, 1000, 140          # 8 key tiles, the last one ragged (104 keys)
    q, k, v = _qkv(B, H, N, N, D, seed=2000 + D)
    idx = _rand_idx(N, kr, seed=2001)
    pad = torch.zeros(B, N)
    for t0 in (0, 2, 3):
        pad[:, t0 * 128:(t0 + 1) * 128] = float("-inf")
    pad[:, 896:] = float("-inf")           # the ragged last tile, all of it
    pad[:, 5 * 128 + 7:5 * 128 + 40] = float("-inf")   # a partly padded live tile
    bias = None
    if bias_kind is not None:
        g = _gen(2002)
        bias = torch.randn(B, 1, N, N, generator=g)
        if bias_kind == "bf16":
            bias = bias.to(BF)
    dv = lambda t: None if t is None else t.to(DEV)
    out = run(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), pad=dv(pad), bias=dv(bias))
    for h in range(H):
        ref = oracle_rows(q, k, v, idx.numpy(), 0, h, pad=pad, bias=bias)
        check_attn(f64(out[0, h]), ref, f"D={D} bias={bias_kind} h{h}")
    vg = v.clone()
    dead = torch.isinf(pad[0])
    vg[:, :, dead] = 1e4
    o2 = run(q.to(DEV), k.to(DEV), vg.to(DEV), idx.to(DEV), pad=dv(pad), bias=dv(bias))
    assert torch.equal(out, o2)


@pytest.mark.parametrize("N", [1024 * 128, 1026 * 128 - 56])
def test_key_tile_skipping_at_its_capacity(N):
    """The live-tile bitmask covers up to 1024 key tiles: at exactly 1024
    tiles the skipping runs with every bitmask word in use (dead tiles first,
    in the middle and last); past that every tile is processed, and the result
    must be the same."""
    B, H, D, kr = 1, 1, 64, 64
    q, k, v = _qkv(B, H, 512, N, D, seed=3000)
    idx = _rand_idx(512, kr, seed=3001)
    nk = (N + 127) // 128
    pad = torch.zeros(B, N)
    for t0 in (0, 500, nk - 1):
        pad[:, t0 * 128:min(N, (t0 + 1) * 128)] = float("-inf")
    out = run(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), pad=pad.to(DEV))
    ref = oracle_rows(q, k, v, idx.numpy(), 0, 0, pad=pad)
    check_attn(f64(out[0, 0]), ref, f"N={N}")


def test_row_constant_mask_elision_is_invisible():
    """A row-constant additive bias (removable by the criterion) changes the
    GPU result only by rounding."""
    B, H, N, D = 1, 2, 512, 96
    q, k, v = _qkv(B, H, N, N, D, seed=21)
    c = (torch.rand(N, 1, generator=_gen(22)) * 8 - 4).expand(N, N)
    bias = c.reshape(1, 1, N, N).contiguous()
    idx = _rand_idx(N, 100, seed=23).to(DEV)
    with_mask = run(q.to(DEV), k.to(DEV), v.to(DEV), idx, bias=bias.to(DEV))
    without = run(q.to(DEV), k.to(DEV), v.to(DEV), idx)
    check_attn(f64(with_mask), f64(without), "elided vs kept row-constant mask")


def test_explicit_scale_and_fully_masked_row_and_bad_index():
    B, H, N, D = 1, 1, 256, 64
    q, k, v = _qkv(B, H, N, N, D, seed=31)
    idx = torch.arange(0, 256, 4, dtype=torch.int32)
    out = run(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), scale=0.3)
    check_attn(f64(out[0, 0]), oracle.attn_subset(f64(q[0, 0]), f64(k[0, 0]), f64(v[0, 0]), idx.numpy(),
                                                  scale=0.3))
    pad = torch.full((1, N), float("-inf"), device=DEV)
    out = run(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), pad=pad, status=sd().ERR_MASKED_ROW)
    assert torch.count_nonzero(out) == 0
    bad = idx.clone()
    bad[5] = N
    out = torch.full((1, 1, idx.numel(), D), 7.0, dtype=BF, device=DEV)
    run(q.to(DEV), k.to(DEV), v.to(DEV), bad.to(DEV), out=out, status=sd().ERR_INDEX)
    assert torch.all(out[0, 0, 5] == 7.0)  # the bad row is skipped


def test_config_1024_full_size():
    w = wl.W1024
    q, k, v = wl.qkv(w, device=DEV)
    idx = _rand_idx(w.N, w.k, seed=41).to(DEV)
    out = run(q, k, v, idx)
    rows = np.arange(0, w.k, 7)
    for (b, h) in [(0, 0), (1, 23), (0, 11)]:
        ref = oracle_rows(q, k, v, idx.cpu().numpy(), b, h, rows=rows)
        check_attn(f64(out[b, h, torch.as_tensor(rows, device=DEV)]), ref, f"b{b}h{h}")


def test_config_2560_srsu_launch_as_benchmarked():
    """The headline workload, in the launch configuration the benchmark
    times: gathered S rows from the partition, scattered into O_state."""
    w = wl.W2560
    q, k, v = wl.qkv(w, device=DEV)
    score = wl.blob_scores(wl.Workload("2560b", 2, B=1, H=1, N=w.N, d=w.d, L=1, n_valid=1,
                                       rho=w.rho, grid=w.grid)).to(DEV)
    idx = torch.empty(w.k, dtype=torch.int32, device=DEV)
    sd().safedit_partition_finalize(score, w.N, w.k, idx, None, None)
    state = torch.zeros(w.B, w.H, w.N, w.d, dtype=BF, device=DEV)
    run(q, k, v, idx, out=state, scattered=True)
    rows = np.linspace(0, w.k - 1, 48).astype(np.int64)
    ic = idx.cpu().numpy()
    for (b, h) in [(0, 0), (1, 17)]:
        ref = oracle_rows(q, k, v, ic, b, h, rows=rows)
        got = state[b, h, torch.as_tensor(ic[rows].astype(np.int64), device=DEV)]
        check_attn(f64(got), ref, f"b{b}h{h}")


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("kind", ["pad", "bias_bf16", "pad+bias_bf16", "bias_f32"])
def test_config_stress_kept_masks_sampled(kind, split):
    """The mask-stress shape in the launch configurations the benchmark times
    (blob-score rows scattered into the state; whole units, and tail-balanced:
    the last 48 units, slices 29..31 from row block 12 of slice 29 on, in 3
    key parts), for every kept-mask variant; sampled rows of a whole-unit head
    and of a split one against the oracle."""
    w = wl.STRESS
    q, k, v = wl.qkv(w, device=DEV)
    score = wl.blob_scores(w).to(DEV)
    idx = torch.empty(w.k, dtype=torch.int32, device=DEV)
    sd().safedit_partition_finalize(score, w.N, w.k, idx, None, None)
    pad = bias = None
    if kind.startswith("pad"):
        pad = torch.zeros(1, w.N, device=DEV)
        pad[:, w.N - w.N // 8:] = float("-inf")   # text-padding style key mask (kept)
    if "bias" in kind:
        bias = wl.mask(w, "bias", device=DEV)     # non-uniform bias (kept), [1,1,N,N] bf16
        if kind.endswith("f32"):
            bias = bias.float()
    state = torch.zeros(w.B, w.H, w.N, w.d, dtype=BF, device=DEV)
    if split:
        _, nbytes = run_ws(q, k, v, idx, pad=pad, bias=bias, out=state, scattered=True)
        assert nbytes == 48 * 3 * 256 * (w.d + 2) * 4
    else:
        run(q, k, v, idx, pad=pad, bias=bias, out=state, scattered=True)
    rows = np.linspace(0, w.k - 1, 24).astype(np.int64)
    ic = idx.cpu().numpy()
    for h in (0, 31):
        ref = oracle_rows(q, k, v, ic, 0, h, rows=rows, pad=pad, bias=bias)
        got = state[0, h, torch.as_tensor(ic[rows].astype(np.int64), device=DEV)]
        check_attn(f64(got), ref, f"{kind} h{h}")


def test_3072_sweep_sampled():
    w = wl.W3072
    q, k, v = wl.qkv(w, device=DEV)
    score = wl.blob_scores(w).to(DEV)
    for rho in w.rho_sweep:
        kk = wl.k_of(rho, w.N)
        idx = torch.empty(kk, dtype=torch.int32, device=DEV)
        sd().safedit_partition_finalize(score, w.N, kk, idx, None, None)
        out = run(q, k, v, idx)
        rows = np.linspace(0, kk - 1, 12).astype(np.int64)
        ref = oracle_rows(q, k, v, idx.cpu().numpy(), 1, 5, rows=rows)
        check_attn(f64(out[1, 5, torch.as_tensor(rows, device=DEV)]), ref, f"rho={rho}")
        del out


def test_compact_query_rows_over_all_keys():
    """Fresh S-row queries given compact ([B,H,k,d], idx = NULL) attend over
    the N-row state: the form an SRSU step takes when only the S rows were
    projected."""
    B, H, N, D, kr = 2, 3, 900, 96, 271
    q, k, v = _qkv(B, H, kr, N, D, seed=91)
    out = run(q.to(DEV), k.to(DEV), v.to(DEV))
    for b in range(B):
        for h in range(H):
            ref = oracle.attn_subset(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]))
            check_attn(f64(out[b, h]), ref, f"b{b}h{h}")


def test_config_2560_dense_anchor_as_benchmarked():
    """The CAR anchor of the headline workload in the launch configuration the
    benchmark times (idx = NULL: all 25600 rows of all 48 slices, output
    [B,H,N,d]); sampled rows of two slices against the oracle's dense
    (matrix-form) attention on those query rows."""
    w = wl.W2560
    q, k, v = wl.qkv(w, device=DEV)
    out = torch.zeros(w.B, w.H, w.N, w.d, dtype=BF, device=DEV)
    run(q, k, v, out=out)
    rows = np.linspace(0, w.N - 1, 64).astype(np.int64)
    rt = torch.as_tensor(rows, device=DEV)
    for (b, h) in [(0, 3), (1, 20)]:
        ref = oracle.attn_dense(f64(q[b, h, rt]), f64(k[b, h]), f64(v[b, h]))
        check_attn(f64(out[b, h, rt]), ref, f"anchor b{b}h{h}")


def run_ws(q, k, v, idx=None, out=None, scattered=False, pad=None, bias=None, status=0):
    """safedit_attn_subset_ws with a workspace of exactly the size the plan asks for."""
    B, H, Nq, D = q.shape
    n = Nq if idx is None else idx.numel()
    nbytes = sd().safedit_attn_subset_workspace_size(B, H, n, k.shape[2], D)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=DEV) if nbytes else None
    if out is None:
        out = torch.zeros(B, H, Nq if scattered else n, D, dtype=BF, device=DEV)
    sd().safedit_attn_subset_ws(q, k, v, idx, n, pad, bias, 0.0, out, int(scattered), ws)
    expect_status(status)
    return out, nbytes


@pytest.mark.parametrize("B,H,Nq,Nk,D,k_rows", [(1, 3, 2000, 2000, 96, 600),    # 9 units -> 4 key parts each
                                                 (1, 2, 700, 4000, 64, 300),     # ragged last key tile in a part
                                                 (2, 3, 900, 1100, 128, None),   # dense rows, d = 128
                                                 (1, 20, 512, 8192, 96, 300),    # 40 units -> 3 parts each
                                                 (1, 50, 700, 4096, 96, 700)])   # 148 whole units + 2 in 4 parts
def test_tail_split_matches_oracle(B, H, Nq, Nk, D, k_rows):
    """The tail-balanced launch: units of 256 query rows run as key-range parts
    whose partial (O, m, l) the merge kernel combines; against the oracle, and
    within the attention tolerance of the whole-unit launch."""
    q, k, v = _qkv(B, H, Nq, Nk, D, seed=3 * Nq + Nk + D)
    idx = None if k_rows is None else _rand_idx(Nq, k_rows, seed=Nk + D)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    idd = None if idx is None else idx.to(DEV)
    out, nbytes = run_ws(qd, kd, vd, idd)
    assert nbytes > 0, "the shape should give a split tail"
    ix = np.arange(Nq, dtype=np.int32) if idx is None else idx.numpy()
    for b in range(B):
        for h in range(0, H, max(1, H // 4)):
            ref = oracle_rows(q, k, v, ix, b, h)
            check_attn(f64(out[b, h]), ref, f"b{b}h{h}")
    whole = run(qd, kd, vd, idd)
    check_attn(f64(out), f64(whole), "split vs whole units")


def test_tail_split_scattered_state_and_errors():
    """Scattered output: the merge writes the S rows at their token index and
    leaves the context rows alone; a workspace smaller than asked for is
    refused before any launch."""
    B, H, N, D, kr = 1, 6, 1500, 96, 500
    q, k, v = _qkv(B, H, N, N, D, seed=1234)
    idx = _rand_idx(N, kr, seed=4321)
    state = torch.randn(B, H, N, D, generator=_gen(99)).to(BF)
    st_d = state.to(DEV)
    _, nbytes = run_ws(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), out=st_d, scattered=True)
    assert nbytes > 0
    keep = torch.ones(N, dtype=torch.bool)
    keep[idx.long()] = False
    assert torch.equal(st_d.cpu()[:, :, keep].view(torch.int16), state[:, :, keep].view(torch.int16))
    for h in (0, 5):
        check_attn(f64(st_d[0, h, idx.long().to(DEV)]), oracle_rows(q, k, v, idx.numpy(), 0, h), f"h{h}")
    small = torch.empty(nbytes - 16, dtype=torch.uint8, device=DEV)
    out = torch.zeros(B, H, kr, D, dtype=BF, device=DEV)
    with pytest.raises(sd().SafeditError) as e:
        sd().safedit_attn_subset_ws(q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV), kr, None, None, 0.0, out, 0,
                                    small)
    assert e.value.code == sd().ERR_INVALID_ARG


@pytest.mark.parametrize("D", [96, 128])
@pytest.mark.parametrize("kind", ["pad", "bias_bf16", "pad_bias_bf16", "bias_f32"])
def test_tail_split_with_kept_masks(D, kind):
    """Kept masks through the tail-balanced launch (9 units of 16 key tiles,
    each in 4 parts of 4 tiles): dead key tiles inside a part and one part
    whose whole key range is padding (its rows leave nothing to the merge),
    max jumps past the lazy-rescale threshold, a ragged last tile; against the
    oracle and within tolerance of the whole-unit launch."""
    B, H, N, kr = 1, 3, 2000, 600          # 16 key tiles, the last one 80 keys
    q, k, v = _qkv(B, H, N, N, D, seed=3000 + D)
    idx = _rand_idx(N, kr, seed=3001)
    pad = bias = None
    if "pad" in kind:
        pad = torch.zeros(B, N)
        pad[:, 512:1024] = float("-inf")    # tiles 4..7: all of part 1
        pad[:, 1536:1664] = float("-inf")   # tile 12: the first tile of part 3
        pad[:, 3::11] = float("-inf")
        pad[:, 1100:1110] += 15.0           # a max jump in part 2
    if "bias" in kind:
        g = _gen(3002 + D)
        bias = torch.randn(B, 1 if "bf16" in kind else H, N, N, generator=g) * 0.5
        bias[..., ::2, 300:310] += 12.0     # part 0
        bias[..., 1::2, 1900:1905] += 14.0  # the ragged tile, part 3
        if "bf16" in kind:
            bias = bias.to(BF)
    dv = lambda t: None if t is None else t.to(DEV)  # noqa: E731
    qd, kd, vd, idd = q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV)
    out, nbytes = run_ws(qd, kd, vd, idd, pad=dv(pad), bias=dv(bias))
    assert nbytes == 9 * 4 * 256 * (D + 2) * 4
    for h in range(H):
        ref = oracle_rows(q, k, v, idx.numpy(), 0, h, pad=pad, bias=bias)
        check_attn(f64(out[0, h]), ref, f"{kind} D={D} h{h}")
    whole = run(qd, kd, vd, idd, pad=dv(pad), bias=dv(bias))
    check_attn(f64(out), f64(whole), "split vs whole units")


def test_tail_split_bad_index_and_explicit_scale():
    """Through the key-range parts and the merge: an out-of-range index sets
    SAFEDIT_ERR_INDEX and its row is skipped (neither written by a part nor
    by the merge); an explicit scale reaches every part."""
    B, H, N, D, kr = 1, 3, 2000, 96, 600     # 9 units in 4 key parts
    q, k, v = _qkv(B, H, N, N, D, seed=5000)
    idx = _rand_idx(N, kr, seed=5001)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    nbytes = sd().safedit_attn_subset_workspace_size(B, H, kr, N, D)
    assert nbytes > 0
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    out = torch.zeros(B, H, kr, D, dtype=BF, device=DEV)
    sd().safedit_attn_subset_ws(qd, kd, vd, idx.to(DEV), kr, None, None, 0.3, out, 0, ws)
    expect_status(0)
    for h in (0, 2):
        check_attn(f64(out[0, h]), oracle_rows(q, k, v, idx.numpy(), 0, h, scale=0.3), f"scale h{h}")
    bad = idx.clone()
    bad[300] = N + 5
    out = torch.full((B, H, kr, D), 7.0, dtype=BF, device=DEV)
    sd().safedit_attn_subset_ws(qd, kd, vd, bad.to(DEV), kr, None, None, 0.0, out, 0, ws)
    expect_status(sd().ERR_INDEX)
    assert torch.all(out[:, :, 300] == 7.0)
    keep = [r for r in range(kr) if r != 300]
    check_attn(f64(out[0, 1, keep]), oracle_rows(q, k, v, idx.numpy(), 0, 1, rows=keep), "other rows")


def test_tail_split_fully_masked_rows():
    """A batch whose every key is padding: no part has an admissible key, so
    the merge reports SAFEDIT_ERR_MASKED_ROW and writes zeros, as the
    whole-unit launch does; the other batch is unaffected."""
    B, H, N, D, kr = 2, 2, 2000, 96, 700   # 3 x 4 = 12 units of 16 key tiles
    q, k, v = _qkv(B, H, N, N, D, seed=4000)
    idx = _rand_idx(N, kr, seed=4001)
    pad = torch.zeros(B, N)
    pad[1] = float("-inf")
    qd, kd, vd, idd = q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV)
    out, nbytes = run_ws(qd, kd, vd, idd, pad=pad.to(DEV), status=sd().ERR_MASKED_ROW)
    assert nbytes > 0
    assert not out[1].any()
    for h in range(H):
        check_attn(f64(out[0, h]), oracle_rows(q, k, v, idx.numpy(), 0, h, pad=pad), f"h{h}")


def test_tail_split_as_benchmarked():
    """The launches the plan splits at the benchmarked sizes: the 1024^2 dense
    anchor (768 units = 5 waves + 28 units in 4 key parts) and the stress-case
    SRSU (640 units = 4 waves + 48 in 3 parts); sampled rows of split units
    and of whole units against the oracle.  The 2560^2 launches keep whole
    units: their predicted saving is under 3% of the launch."""
    w = wl.W1024
    q, k, v = wl.qkv(w, device=DEV)
    out = torch.zeros(w.B, w.H, w.N, w.d, dtype=BF, device=DEV)
    _, nbytes = run_ws(q, k, v, None, out=out)
    assert nbytes == 28 * 4 * 256 * (w.d + 2) * 4
    # units are (row block, slice) with row blocks fastest: the last 28 are
    # row blocks 4..15 of slice 46 (b = 1, h = 22) and all of slice 47
    rows = np.linspace(0, w.N - 1, 48).astype(np.int64)
    rt = torch.as_tensor(rows, device=DEV)
    for (b, h) in [(1, 23), (1, 22), (0, 5)]:
        ref = oracle.attn_dense(f64(q[b, h, rt]), f64(k[b, h]), f64(v[b, h]))
        check_attn(f64(out[b, h, rt]), ref, f"anchor b{b}h{h}")
    assert sd().safedit_attn_subset_workspace_size(wl.W2560.B, wl.W2560.H, wl.W2560.k, wl.W2560.N, 96) == 0
    del q, k, v, out
    w = wl.STRESS
    q, k, v = wl.qkv(w, device=DEV)
    idx = torch.empty(w.k, dtype=torch.int32, device=DEV)
    sd().safedit_partition_finalize(wl.blob_scores(w, device=DEV).contiguous(), w.N, w.k, idx, None, None)
    state = torch.zeros(w.B, w.H, w.N, w.d, dtype=BF, device=DEV)
    _, nbytes = run_ws(q, k, v, idx, out=state, scattered=True)
    assert nbytes == 48 * 3 * 256 * (w.d + 2) * 4
    # the last 48 units: row blocks 12..19 of slice 29, all of slices 30 and 31
    ic = idx.cpu().numpy()
    rows = np.linspace(0, w.k - 1, 40).astype(np.int64)
    for h in (31, 29, 3):
        ref = oracle_rows(q, k, v, ic, 0, h, rows=rows)
        got = state[0, h, torch.as_tensor(ic[rows].astype(np.int64), device=DEV)]
        check_attn(f64(got), ref, f"stress h{h}")
