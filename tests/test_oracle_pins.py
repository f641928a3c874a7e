"""Pins of the fp64 CPU oracle against things other than itself: closed forms,
hand-derived fixtures, brute force on tiny inputs, invariants the pages state,
and library routines (torch float64 softmax / SDPA, numpy einsum) for the cases
that reduce to them.  Each test names the passage it follows.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(20261202)


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------------------
# Attention (C6): SAFE-DiT summary, 방법론 3 (SRSU / CAR); AccelAes B.2.
# ---------------------------------------------------------------------------
def test_subset_rows_equal_dense_rows():
    """An S row attends to the global K/V, so it equals the same row of the
    dense (anchor) attention [SAFE-DiT summary, 방법론 3]."""
    Nq, N, d = 67, 53, 12
    q, k, v = rng.standard_normal((Nq, d)), rng.standard_normal((N, d)), rng.standard_normal((N, d))
    idx = np.sort(rng.choice(Nq, size=23, replace=False)).astype(np.int32)
    dense = oracle.attn_dense(q, k, v)
    sub = oracle.attn_subset(q, k, v, idx)
    assert np.abs(sub - dense[idx]).max() <= 1e-13
    ident = oracle.attn_subset(q, k, v, np.arange(Nq, dtype=np.int32))
    assert np.abs(ident - dense).max() <= 1e-13


def test_attention_matches_torch_sdpa_float64():
    """Library routine: torch SDPA in float64 with an additive mask (key
    padding + non-uniform bias), scale 1/sqrt(d) and a custom scale."""
    Nq, N, d = 40, 70, 16
    q, k, v = rng.standard_normal((Nq, d)), rng.standard_normal((N, d)), rng.standard_normal((N, d))
    pad = np.where(rng.random(N) < 0.2, -np.inf, 0.0)
    pad[0] = 0.0
    bias = rng.standard_normal((Nq, N))
    for scale in (None, 0.37):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None],
            attn_mask=torch.tensor(pad[None, :] + bias)[None],
            scale=scale).numpy()[0]
        dense = oracle.attn_dense(q, k, v, pad=pad, bias=bias, scale=scale)
        idx = np.arange(Nq, dtype=np.int32)[::3].copy()
        sub = oracle.attn_subset(q, k, v, idx, pad=pad, bias_rows=bias[idx], scale=scale)
        assert np.abs(dense - ref).max() <= 1e-12
        assert np.abs(sub - ref[idx]).max() <= 1e-12
    # transposed operand / wrong scale would fail this: check the scale is used
    ref1 = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None]).numpy()[0]
    assert np.abs(oracle.attn_dense(q, k, v, scale=0.9) - ref1).max() > 1e-3


def test_row_constant_shift_is_invisible():
    """An additive mask that shifts each row by a constant c_i does not change
    softmax outputs [SAFE-DiT summary, 방법론 1; Italian page, Metodologia 1]."""
    Nq, N, d = 33, 41, 8
    q, k, v = rng.standard_normal((Nq, d)), rng.standard_normal((N, d)), rng.standard_normal((N, d))
    base = oracle.attn_dense(q, k, v)
    c = rng.uniform(-4, 4, size=(Nq, 1)) * np.ones((1, N))
    assert np.abs(oracle.attn_dense(q, k, v, bias=c) - base).max() <= 1e-13
    idx = np.arange(0, Nq, 2, dtype=np.int32)
    assert np.abs(oracle.attn_subset(q, k, v, idx, bias_rows=c[idx]) - base[idx]).max() <= 1e-13
    zero = np.zeros((Nq, N))
    assert np.array_equal(oracle.attn_dense(q, k, v, bias=zero), base)
    # a non-uniform bias is not a shift: it must change the output
    assert np.abs(oracle.attn_dense(q, k, v, bias=rng.standard_normal((Nq, N))) - base).max() > 1e-3


def test_padding_keys_get_exactly_zero_weight_in_attention():
    """Kept semantic masks [SAFE-DiT summary, 방법론 1 보존]: a -inf padded key
    contributes exactly nothing; bit-identical to removing the key."""
    Nq, N, d, n_pad = 20, 48, 8, 11
    q, k, v = rng.standard_normal((Nq, d)), rng.standard_normal((N, d)), rng.standard_normal((N, d))
    pad = np.zeros(N)
    pad[N - n_pad:] = -np.inf
    with_pad = oracle.attn_subset(q, k, v, pad=pad)
    removed = oracle.attn_subset(q, k[: N - n_pad], v[: N - n_pad])
    assert np.array_equal(with_pad, removed)
    v2 = v.copy()
    v2[N - n_pad:] = 1e30  # garbage in padded values must not leak
    assert np.array_equal(oracle.attn_subset(q, k, v2, pad=pad), removed)


def test_attention_closed_forms():
    d = 5
    # one key: output is that value row
    q, k, v = rng.standard_normal((3, d)), rng.standard_normal((1, d)), rng.standard_normal((1, d))
    assert np.array_equal(oracle.attn_subset(q, k, v), np.repeat(v, 3, axis=0))
    # all-equal logits (q = 0): output is the mean of V
    N = 37
    k, v = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    out = oracle.attn_dense(np.zeros((2, d)), k, v)
    assert np.abs(out - v.mean(axis=0)).max() <= 1e-14
    # d = 1, two keys: logistic weights
    qs, k2, v2 = 0.7, np.array([[1.5], [-0.5]]), np.array([[2.0], [-3.0]])
    w1 = 1.0 / (1.0 + math.exp(-(qs * (1.5 - (-0.5)) * 0.8)))
    out = oracle.attn_subset(np.array([[qs]]), k2, v2, scale=0.8)
    assert abs(out[0, 0] - (w1 * 2.0 + (1 - w1) * (-3.0))) <= 1e-15


def test_fully_masked_row_is_an_error():
    q, k, v = np.ones((2, 3)), np.ones((4, 3)), np.ones((4, 3))
    with pytest.raises(oracle.OracleError):
        oracle.attn_subset(q, k, v, pad=np.full(4, -np.inf))
    with pytest.raises(oracle.OracleError):
        oracle.attn_dense(q, k, v, pad=np.full(4, -np.inf))
    with pytest.raises(oracle.OracleError):
        oracle.attn_subset(q, k, v, idx=np.array([2], dtype=np.int32))


# ---------------------------------------------------------------------------
# Cross-attention probabilities (C1): SAFE-DiT summary 방법론 2; AccelAes B.1.
# ---------------------------------------------------------------------------
def test_cross_attn_probs_padding_and_softmax():
    H, N, L, d, nv = 3, 17, 12, 8, 7
    q, k = rng.standard_normal((H, N, d)), rng.standard_normal((H, L, d))
    valid = np.zeros(L, dtype=np.uint8)
    valid[:nv] = 1
    P = oracle.cross_attn_probs(q, k, valid)
    assert np.all(P[:, :, nv:] == 0.0)
    assert np.abs(P.sum(-1) - 1.0).max() <= 1e-14
    # library routine: float64 softmax over the valid keys
    logits = torch.einsum("hnd,hld->hnl", torch.tensor(q), torch.tensor(k[:, :nv])) / math.sqrt(d)
    ref = torch.softmax(logits, dim=-1).numpy()
    assert np.abs(P[:, :, :nv] - ref).max() <= 1e-15
    # the padded tail physically removed gives bit-identical probabilities
    P2 = oracle.cross_attn_probs(q, k[:, :nv], valid[:nv])
    assert np.array_equal(P[:, :, :nv], P2)
    # non-prefix padding pattern
    valid3 = (rng.random(L) < 0.5).astype(np.uint8)
    valid3[3] = 1
    P3 = oracle.cross_attn_probs(q, k, valid3)
    assert np.all(P3[:, :, valid3 == 0] == 0.0)
    with pytest.raises(oracle.OracleError):
        oracle.cross_attn_probs(q, k, np.zeros(L, dtype=np.uint8))


# ---------------------------------------------------------------------------
# Partition (C2-C4): SAFE-DiT summary 방법론 2; AccelAes B.1 step 4.
# ---------------------------------------------------------------------------
def test_accumulate_matches_einsum_and_content_selection():
    H, N, L = 4, 29, 10
    P = rng.random((H, N, L))
    content = (rng.random(L) < 0.6).astype(np.uint8)
    start = rng.random(N)
    got = oracle.partition_accumulate(P, content, start)
    ref = start + np.einsum("hnl,l->n", P, content.astype(np.float64))
    assert np.abs(got - ref).max() <= 1e-13
    # only content positions count: changing a non-content column changes nothing
    P2 = P.copy()
    P2[:, :, content == 0] += 5.0
    assert np.array_equal(oracle.partition_accumulate(P2, content, start), got)
    # accumulation over calls adds up
    twice = oracle.partition_accumulate(P, content, got)
    assert np.abs(twice - (start + 2 * (ref - start))).max() <= 1e-12


def _brute_topk(score, k):
    """Exhaustive: the k-subset with the largest score multiset, ties broken
    by the lexicographically smallest index set."""
    best, best_key = None, None
    n = len(score)
    for comb in itertools.combinations(range(n), k):
        key = (sorted((score[i] for i in comb), reverse=True), [-i for i in comb])
        if best is None or key > best_key:
            best, best_key = comb, key
    return list(best)


def test_partition_select_brute_force_tiny():
    for trial in range(60):
        n = int(rng.integers(1, 11))
        k = int(rng.integers(0, n + 1))
        # integer-valued scores to force ties at the threshold
        score = rng.integers(0, 4, size=n).astype(np.float64)
        idx_s, idx_c, _ = oracle.partition_select(score, k)
        assert list(idx_s) == _brute_topk(list(score), k)
        assert sorted(list(idx_s) + list(idx_c)) == list(range(n))
        assert list(idx_c) == sorted(idx_c)


def test_partition_select_against_python_sort():
    for n in (37, 256):
        for dup in (False, True):
            score = rng.random(n)
            if dup:
                score = np.round(score * 8) / 8
            for k in (0, 1, n // 4, n // 2, n - 1, n):
                order = sorted(range(n), key=lambda i: (-score[i], i))
                idx_s, idx_c, s = oracle.partition_select(score, k)
                assert list(idx_s) == sorted(order[:k])
                assert list(idx_c) == sorted(order[k:])
                lo, hi = score.min(), score.max()
                assert np.array_equal(s, ((score - lo) / (hi - lo)).astype(np.float32))


def test_partition_hand_fixture():
    for ln in _lines("partition_hand.txt"):
        kk, sc, exp_s, exp_sv = [x.strip() for x in ln.split("|")]
        score = np.array([float(x) for x in sc.split()])
        exp_idx = [] if exp_s == "-" else [int(x) for x in exp_s.split()]
        idx_s, idx_c, s = oracle.partition_select(score, int(kk))
        assert list(idx_s) == exp_idx, ln
        assert np.array_equal(s, np.array([float(x) for x in exp_sv.split()], dtype=np.float32)), ln


def test_partition_s_is_minmax_and_affine_invariant():
    score = rng.random(100) * 3 + 1
    idx_s, _, s = oracle.partition_select(score, 30)
    assert s[np.argmax(score)] == 1.0 and s[np.argmin(score)] == 0.0
    assert np.all((s >= 0) & (s <= 1))
    idx2, _, s2 = oracle.partition_select(score * 2.5 + 7.0, 30)
    assert np.array_equal(idx_s, idx2)
    assert np.abs(s - s2).max() <= 1e-6
    with pytest.raises(oracle.OracleError):
        oracle.partition_select(np.array([1.0, np.nan]), 1)


# ---------------------------------------------------------------------------
# Mask elision (C5): SAFE-DiT summary 방법론 1.
# ---------------------------------------------------------------------------
def test_mask_criterion_hand_fixture():
    rows, expect = [], []
    for ln in _lines("mask_rows_hand.txt"):
        e, vals = ln.split("|")
        expect.append(int(e))
        rows.append([float(x) for x in vals.split()])
    m = np.array(rows)
    verdict, flags = oracle.mask_row_constant(m)
    assert list(flags) == expect
    assert verdict == 0
    good = m[np.array(expect) == 1]
    assert oracle.mask_row_constant(good)[0] == 1


def test_mask_criterion_dtypes_and_bool():
    # bf16 and fp16 row-constant masks widen exactly
    c = torch.tensor(rng.uniform(-4, 4, size=(6, 1))).expand(6, 9)
    for dt in (torch.bfloat16, torch.float16, torch.float32):
        v, f = oracle.mask_row_constant(c.to(dt).contiguous())
        assert v == 1 and f.all()
    bm = torch.ones((3, 4, 10), dtype=torch.bool)
    v, f = oracle.mask_row_constant(bm)
    assert v == 1 and f.shape == (3, 4) and f.all()
    bm[1, 2, 7] = False
    v, f = oracle.mask_row_constant(bm)
    assert v == 0 and f[1, 2] == 0 and f.sum() == 11
    v, f = oracle.mask_row_constant(torch.zeros((1, 5), dtype=torch.bool))
    assert v == 0  # all False: fully masked, not a shift


# ---------------------------------------------------------------------------
# Scatter / gather (C7): SAFE-DiT summary 방법론 3 (cached context state).
# ---------------------------------------------------------------------------
def test_scatter_gather_identities():
    N, d = 50, 6
    state = rng.standard_normal((N, d)).astype(np.float32)
    fresh = rng.standard_normal((N, d)).astype(np.float32)
    idx = np.sort(rng.choice(N, size=17, replace=False)).astype(np.int32)
    # gather o scatter = id on S
    merged = oracle.scatter_rows(fresh[idx], state, idx)
    assert np.array_equal(oracle.gather_rows(merged, idx), fresh[idx])
    # S rows from fresh, C rows from the cache
    expect = state.copy()
    expect[idx] = fresh[idx]
    assert np.array_equal(merged, expect)
    cidx = np.setdiff1d(np.arange(N), idx).astype(np.int32)
    assert np.array_equal(oracle.gather_rows(merged, cidx), state[cidx])
    with pytest.raises(oracle.OracleError):
        oracle.scatter_rows(fresh[:2], state, np.array([3, 3], dtype=np.int32))
    with pytest.raises(oracle.OracleError):
        oracle.scatter_rows(fresh[:1], state, np.array([N], dtype=np.int32))
    with pytest.raises(oracle.OracleError):
        oracle.gather_rows(state, np.array([-1], dtype=np.int32))


# ---------------------------------------------------------------------------
# SW-CFG (C8): SAFE-DiT summary 방법론 4; AccelAes B.2 spatial CFG.
# ---------------------------------------------------------------------------
def test_sw_cfg_hand_fixture():
    rows = np.array([[float(x) for x in ln.split()] for ln in _lines("sw_cfg_hand.txt")])
    s, c, u, g, out = rows.T
    got = oracle.sw_cfg(c[:, None], u[:, None], s, 3.0, 5.0)
    assert np.array_equal(got[:, 0], out)


def test_sw_cfg_special_cases():
    N, F = 31, 16
    c = rng.standard_normal((N, F)).astype(np.float32)
    u = rng.standard_normal((N, F)).astype(np.float32)
    s = rng.random(N).astype(np.float32)
    assert np.abs(oracle.sw_cfg(c, u, s, 1.0, 1.0) - c).max() <= 1e-15
    assert np.array_equal(oracle.sw_cfg(c, u, s, 0.0, 0.0), u.astype(np.float64))
    sb = (rng.random(N) < 0.5).astype(np.float32)  # AccelAes binary focus map
    got = oracle.sw_cfg(c, u, sb, 2.0, 7.5)
    gam = np.where(sb > 0, 7.5, 2.0)[:, None]
    assert np.abs(got - (u + gam * (c.astype(np.float64) - u))).max() <= 1e-14


# ---------------------------------------------------------------------------
# Schedule (C9): SAFE-DiT summary 방법론 2-3 (warm-up, fixed split, SRSU/CAR).
# ---------------------------------------------------------------------------
def _tiny_steps(B, H, N, d, L, k, steps, same_kv):
    out = []
    for t in range(steps):
        q, kf, vf = rng.standard_normal((B, H, N, d)), rng.standard_normal((B, H, N, d)), \
            rng.standard_normal((B, H, N, d))
        if same_kv:  # every step sees the same K/V: the cached context is never stale
            kf, vf = out[0]["k_full"] if out else kf, out[0]["v_full"] if out else vf
        out.append(dict(q=q, k_full=kf, v_full=vf, k_s=None, v_s=None,
                        q_img=rng.standard_normal((B, H, N, d)), k_txt=rng.standard_normal((B, H, L, d)),
                        key_valid=np.ones((B, L), dtype=np.uint8), content=np.ones(L, dtype=np.uint8),
                        eps_c=rng.standard_normal((N, 4)), eps_u=rng.standard_normal((N, 4))))
    return out


def test_trajectory_srsu_rows_equal_dense_when_context_is_fresh():
    """If the cached context equals the current K/V, an SRSU step's S rows are
    the dense anchor's rows (S queries attend to the global K/V), and C rows
    keep the previous anchor's output."""
    B, H, N, d, L, k = 1, 2, 40, 8, 6, 12
    steps = _tiny_steps(B, H, N, d, L, k, 3, same_kv=True)
    warm = oracle.trajectory(steps[:1], 1, 5, k, 2.0, 4.0)
    idx = warm["idx_s"]
    for st in steps:
        st["k_s"] = st["k_full"][:, :, idx]
        st["v_s"] = st["v_full"][:, :, idx]
    res = oracle.trajectory(steps[:2], 1, 5, k, 2.0, 4.0)  # t=0 anchor, t=1 SRSU
    for h in range(H):
        dense1 = oracle.attn_dense(steps[1]["q"][0, h], steps[1]["k_full"][0, h], steps[1]["v_full"][0, h])
        dense0 = oracle.attn_dense(steps[0]["q"][0, h], steps[0]["k_full"][0, h], steps[0]["v_full"][0, h])
        assert np.abs(res["o_state"][0, h][idx] - dense1[idx]).max() <= 1e-13
        c = np.setdiff1d(np.arange(N), idx)
        assert np.array_equal(res["o_state"][0, h][c], dense0[c])
    # guidance: global before the split exists, sensitivity-weighted after it
    s = res["s"].astype(np.float64)
    g = 2.0 + 2.0 * s
    u, cc = steps[1]["eps_u"], steps[1]["eps_c"]
    assert np.abs(res["cfg"][1] - (u + g[:, None] * (cc - u))).max() <= 1e-14
    assert np.abs(res["cfg"][0] - (steps[0]["eps_u"] + 2.0 * (steps[0]["eps_c"] - steps[0]["eps_u"]))).max() <= 1e-14


def test_trajectory_anchor_refreshes_everything():
    B, H, N, d, L, k = 1, 1, 24, 4, 5, 6
    steps = _tiny_steps(B, H, N, d, L, k, 3, same_kv=False)
    for st in steps:
        st["k_s"] = rng.standard_normal((B, H, k, d))
        st["v_s"] = rng.standard_normal((B, H, k, d))
    res = oracle.trajectory(steps, 1, 2, k, 1.0, 1.0)  # t=0 anchor, t=1 SRSU, t=2 anchor
    assert np.array_equal(res["k_state"], steps[2]["k_full"])
    dense = oracle.attn_dense(steps[2]["q"][0, 0], steps[2]["k_full"][0, 0], steps[2]["v_full"][0, 0])
    assert np.array_equal(res["o_state"][0, 0], dense)


# ---------------------------------------------------------------------------
# StepCache (C10): AccelAes summary B.3 (linear extrapolation between full steps).
# ---------------------------------------------------------------------------
def test_stepcache_extrapolation_closed_forms():
    N, F = 23, 8
    c_a, c_b, u_a, u_b = (rng.standard_normal((N, F)) for _ in range(4))
    s = rng.random(N)
    # w = 0 reuses the last full step, w = -1 the one before: the plain combine of that step
    assert np.abs(oracle.stepcache_sw_cfg(c_a, c_b, u_a, u_b, s, 0.0, 3.0, 5.0)
                  - oracle.sw_cfg(c_b, u_b, s, 3.0, 5.0)).max() <= 1e-14
    assert np.abs(oracle.stepcache_sw_cfg(c_a, c_b, u_a, u_b, s, -1.0, 3.0, 5.0)
                  - oracle.sw_cfg(c_a, u_a, s, 3.0, 5.0)).max() <= 1e-14
    # predictions linear in t are reproduced exactly at any later t
    slope_c, slope_u = rng.standard_normal((N, F)), rng.standard_normal((N, F))
    t_a, t_b, t = 10.0, 12.0, 15.0
    ca, cb, ct = c_b + slope_c * t_a, c_b + slope_c * t_b, c_b + slope_c * t
    ua, ub, ut = u_b + slope_u * t_a, u_b + slope_u * t_b, u_b + slope_u * t
    w = (t - t_b) / (t_b - t_a)
    assert np.abs(oracle.stepcache_sw_cfg(ca, cb, ua, ub, s, w, 3.0, 5.0)
                  - oracle.sw_cfg(ct, ut, s, 3.0, 5.0)).max() <= 1e-12


# ---------------------------------------------------------------------------
# SkipSparse FFN caching (C11): AccelAes summary B.2.
# ---------------------------------------------------------------------------
def test_ffn_cached_against_library_and_cache_rule():
    N, D, F = 37, 16, 40
    x = rng.standard_normal((N, D))
    w1, b1 = rng.standard_normal((F, D)) / 4, rng.standard_normal(F)
    w2, b2 = rng.standard_normal((D, F)) / 6, rng.standard_normal(D)
    cache = rng.standard_normal((N, D))
    idx = np.sort(rng.choice(N, size=11, replace=False)).astype(np.int32)
    y = oracle.ffn_cached(x, idx, w1, b1, w2, b2, cache, act=1)
    # library routine: torch's tanh-approximate GELU and float64 matmuls
    xt = torch.tensor(x[idx])
    h = torch.nn.functional.gelu(xt @ torch.tensor(w1).T + torch.tensor(b1), approximate="tanh")
    ref = (h @ torch.tensor(w2).T + torch.tensor(b2)).numpy()
    assert np.abs(y[idx] - ref).max() <= 1e-12
    keep = np.setdiff1d(np.arange(N), idx)
    assert np.array_equal(y[keep], cache[keep])  # background rows reuse the cache
    # no activation: the block is affine, so it is a single matrix
    y0 = oracle.ffn_cached(x, None, w1, None, w2, None, cache, act=0)
    assert np.abs(y0 - x @ (w2 @ w1).T).max() <= 1e-12
    with pytest.raises(oracle.OracleError):
        oracle.ffn_cached(x, np.array([1, 1], dtype=np.int32), w1, b1, w2, b2, cache)


def test_linear_act_against_library_and_closed_forms():
    M, K, N = 23, 19, 31
    a = rng.standard_normal((M, K))
    w, b = rng.standard_normal((N, K)) / 3, rng.standard_normal(N)
    out = oracle.linear_act(a, w, b, act=1)
    ref = torch.nn.functional.gelu(torch.nn.functional.linear(torch.tensor(a), torch.tensor(w), torch.tensor(b)),
                                   approximate="tanh").numpy()
    assert np.abs(out - ref).max() <= 1e-12
    # identity weights, no bias, no activation: the input itself
    assert np.array_equal(oracle.linear_act(a, np.eye(K), None, act=0), a)
    # GELU closed forms: gelu(0) = 0, odd part x/2, gelu(x) -> x for large x, -> 0 for very negative x
    z = oracle.linear_act(np.array([[0.0], [1.0], [-1.0], [12.0], [-12.0]]), np.ones((1, 1)), None, act=1)[:, 0]
    assert z[0] == 0.0
    assert abs((z[1] - z[2]) - 1.0) <= 1e-15  # gelu(x) - gelu(-x) = x
    assert abs(z[3] - 12.0) <= 1e-12 and abs(z[4]) <= 1e-12
    # 0.5 (1 + tanh(sqrt(2/pi) (1 + 0.044715))) at x = 1, from math.tanh directly
    assert abs(z[1] - 0.5 * (1 + math.tanh(math.sqrt(2 / math.pi) * 1.044715))) <= 1e-15
    # the block of C11 is two such projections
    x = rng.standard_normal((7, K))
    w2, b2 = rng.standard_normal((K, N)) / 5, rng.standard_normal(K)
    y = oracle.ffn_cached(x, None, w, b, w2, b2, np.zeros((7, K)), act=1)
    assert np.abs(y - oracle.linear_act(oracle.linear_act(x, w, b, 1), w2, b2, 0)).max() <= 1e-12
