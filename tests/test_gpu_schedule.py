"""A whole tiny trajectory (SAFE-DiT summary, 방법론 2-4) through the C ABI
against the same schedule composed from oracle functions: two dense warm-up
steps feeding the PCSP score, the S/C split, one SRSU step (fresh S-row K/V
scattered into the cached state, subset attention scattered into O_state)
and one dense anchor step, with the guidance combine after every step."""
import numpy as np
import pytest
import torch

import oracle
from spatially_adaptive_dit_b200 import workloads as wl
from tests.gpu_util import CFG_REL, check_attn, expect_status, sd

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(w):
    steps = []
    for t in range(w.steps):
        q, kf, vf = wl.qkv(w, step=t)
        k_s, v_s = wl.fresh_sensitive_kv(w, w.k, step=t)
        q_img, k_txt, valid, content = wl.text(w, step=t)
        eps_c, eps_u = wl.cfg_preds(w, step=t)
        steps.append(dict(q=q, k_full=kf, v_full=vf, k_s=k_s, v_s=v_s, q_img=q_img, k_txt=k_txt,
                          key_valid=valid, content=content, eps_c=eps_c, eps_u=eps_u))
    return steps


def _gpu_trajectory(w, steps):
    S = sd()
    score = torch.zeros(w.N, dtype=torch.float64, device=DEV)
    idx_s = torch.empty(w.k, dtype=torch.int32, device=DEV)
    idx_c = torch.empty(w.N - w.k, dtype=torch.int32, device=DEV)
    s = torch.zeros(w.N, device=DEV)
    P = torch.empty(w.H, w.N, w.L, device=DEV)
    k_state = v_state = o_state = None
    cfg = []
    for t, st in enumerate(steps):
        d = {n: v.to(DEV) for n, v in st.items()}
        if t < w.warmup:
            S.safedit_cross_attn_probs(d["q_img"], d["k_txt"], d["key_valid"], 0, 0.0, P)
            S.safedit_partition_accumulate(P, d["content"], score)
        if t == w.warmup - 1:
            S.safedit_partition_finalize(score, w.N, w.k, idx_s, idx_c, s)
        if oracle.is_anchor_step(t, w.warmup, w.period):
            k_state, v_state = d["k_full"].clone(), d["v_full"].clone()
            o_state = torch.empty_like(d["q"])
            S.safedit_attn_subset(d["q"], k_state, v_state, None, 0, None, None, 0.0, o_state, 0)
        else:
            S.safedit_scatter_state([d["k_s"], d["v_s"]], [k_state, v_state], idx_s, w.k)
            S.safedit_attn_subset(d["q"], k_state, v_state, idx_s, w.k, None, None, 0.0, o_state, 1)
        out = torch.empty_like(d["eps_c"])
        g_sens = w.gamma_sens if t >= w.warmup else w.gamma_ctx
        S.safedit_sw_cfg(d["eps_c"], d["eps_u"], s, w.gamma_ctx, g_sens, out)
        cfg.append(out.cpu())
    expect_status(0)
    return dict(idx_s=idx_s.cpu().numpy(), s=s.cpu().numpy(), score=score.cpu().numpy(),
                k_state=k_state.cpu(), v_state=v_state.cpu(), o_state=o_state.cpu(), cfg=cfg)


@pytest.mark.parametrize("w", [wl.TINY, wl.Workload("tiny96", 5, B=2, H=3, N=640, d=96, L=64, n_valid=40,
                                                     rho=wl.Fraction(3, 10), grid=0, warmup=1, period=3,
                                                     steps=5)])
def test_tiny_trajectory_matches_oracle_schedule(w):
    steps = _inputs(w)
    gpu = _gpu_trajectory(w, steps)
    ref = oracle.trajectory(steps, w.warmup, w.period, w.k, w.gamma_ctx, w.gamma_sens)
    # the GPU aggregates its own fp32 probabilities (bf16 inputs, fp32 MMA and
    # exponentials), the oracle its fp64 ones: the scores agree to ~1e-7
    assert np.abs(gpu["score"] - ref["score"]).max() <= 1e-5 * np.abs(ref["score"]).max()
    # the split: exact except tokens within 1e-6 relative of the threshold score
    tau = np.sort(ref["score"])[::-1][w.k - 1]
    near = set(np.nonzero(np.abs(ref["score"] - tau) <= 1e-6 * abs(tau))[0].tolist())
    assert set(gpu["idx_s"].tolist()) - near == set(ref["idx_s"].tolist()) - near
    # with these seeds no score lies within rounding of the threshold, so the
    # splits agree exactly and the states can be compared row for row
    assert np.array_equal(gpu["idx_s"], ref["idx_s"])
    bf = torch.bfloat16
    assert np.array_equal(gpu["k_state"].view(torch.int16).numpy(),
                          torch.tensor(ref["k_state"]).to(bf).view(torch.int16).numpy())
    for b in range(w.B):
        for h in range(w.H):
            check_attn(gpu["o_state"][b, h].double().numpy(), ref["o_state"][b, h], f"b{b}h{h}")
    for t in range(w.steps):
        c, u = steps[t]["eps_c"].double().numpy(), steps[t]["eps_u"].double().numpy()
        g = np.abs(c - u) * max(w.gamma_ctx, w.gamma_sens) + np.abs(u)
        assert np.all(np.abs(gpu["cfg"][t].double().numpy() - ref["cfg"][t]) <= CFG_REL * g + 1e-30)


@pytest.mark.parametrize("pcsp", ["fused", "unfused"])
def test_head_sharded_trajectory_split_matches_unsharded(pcsp):
    """The benchmark's head-sharded path on one GPU: two trajectories of the
    1024^2 workload keep heads [0, 12) and [12, 24) of the same seeded
    generation; the second one's PCSP score (its heads only) is added to the
    first one's through the reduce hook, standing in for the all-reduce,
    before the split.  The summed score and the S/C split must equal those of
    the unsharded trajectory (the two sums differ only in the order of fp64
    additions), and each shard's attention output must equal the unsharded
    output on its heads."""
    import bench
    w = wl.W1024
    dev = torch.device(DEV)
    stream = torch.cuda.Stream()
    full = bench.Trajectory(w, dev, pcsp=pcsp)
    with torch.cuda.stream(stream):
        full.run(stream)
    stream.synchronize()
    taken = {}
    hi = bench.Trajectory(w, dev, heads=(12, 24), reduce_score=lambda s: taken.setdefault("hi", s.clone()), pcsp=pcsp)
    with torch.cuda.stream(stream):
        hi.run(stream)
    stream.synchronize()
    lo = bench.Trajectory(w, dev, heads=(0, 12), reduce_score=lambda s: s.add_(taken["hi"]), pcsp=pcsp)
    with torch.cuda.stream(stream):
        lo.run(stream)
    stream.synchronize()
    expect_status(0)
    sf, sl = full.score.cpu().numpy(), lo.score.cpu().numpy()
    assert np.abs(sl - sf).max() <= 1e-12 * np.abs(sf).max()
    tau = np.sort(sf)[::-1][w.k - 1]
    near = set(np.nonzero(np.abs(sf - tau) <= 1e-6 * abs(tau))[0].tolist())
    assert set(lo.idx_s.cpu().tolist()) - near == set(full.idx_s.cpu().tolist()) - near
    if not near:
        assert torch.equal(lo.idx_s, full.idx_s)
        assert torch.equal(lo.o_state, full.o_state[:, :12])


def test_guidance_branch_sharded_trajectory_matches_unsharded():
    """The benchmark's guidance-branch split on one GPU: two trajectories of
    the 1024^2 workload keep batch entry 0 (cond) and 1 (uncond) of the same
    seeded generation; only the cond one scores the tokens, the uncond one
    takes its split through the share hook, and each takes the other's
    branch prediction through the exchange hook (standing in for the
    broadcast and the all-gather).  Split and guided output must equal the
    unsharded trajectory's exactly, each branch's state rows bit for bit, and
    its attention output within the attention tolerance (the two launch
    shapes may take different tail-balancing plans)."""
    import bench
    w = wl.W1024
    dev = torch.device(DEV)
    stream = torch.cuda.Stream()
    full = bench.Trajectory(w, dev)
    with torch.cuda.stream(stream):
        full.run(stream)
    stream.synchronize()
    br = {}

    def share(tr):
        if tr.branch == 1:
            for name in ("idx_s", "idx_c", "s"):
                getattr(tr, name).copy_(getattr(br[0], name))

    def exchange(tr):
        tr.eps_c.copy_(br[0].eps_own)
        tr.eps_u.copy_(br[1].eps_own)

    for b in (0, 1):
        br[b] = bench.Trajectory(w, dev, branch=b, share_split=share, exchange_eps=exchange)
    for b in (0, 1):
        with torch.cuda.stream(stream):
            br[b].run(stream)
        stream.synchronize()
    expect_status(0)
    for b in (0, 1):
        assert torch.equal(br[b].idx_s, full.idx_s) and torch.equal(br[b].s, full.s)
        assert torch.equal(br[b].cfg_out, full.cfg_out)
        assert torch.equal(br[b].k_state, full.k_state[b:b + 1])
        check_attn(br[b].o_state.double().cpu().numpy(), full.o_state[b:b + 1].double().cpu().numpy(), f"branch {b}")


def test_guidance_branch_sharded_e2e_leg_matches_unsharded():
    """The benchmark's end-to-end leg (inputs uploaded every step from pinned
    host memory) in the guidance-branch split, on one GPU: each branch
    uploads only its own prediction and takes the other's through the
    exchange hook; the uncond branch uploads no text and takes the split
    through the share hook.  The guided output and the split must equal
    those of the unsharded end-to-end leg exactly, and each branch uploads
    less than the unsharded leg."""
    import types
    import bench
    w = wl.W1024
    dev = torch.device(DEV)
    stream = torch.cuda.Stream()
    args = types.SimpleNamespace(steps=1)
    full = bench.Trajectory(w, dev)
    r_full = bench.run_e2e(full, stream, args)
    torch.cuda.synchronize()
    br = {}

    def share(tr):
        if tr.branch == 1:
            for name in ("idx_s", "idx_c", "s"):
                getattr(tr, name).copy_(getattr(br[0], name))

    def exchange(tr):
        tr.eps_c.copy_(br[0].eps_own)
        tr.eps_u.copy_(br[1].eps_own)

    for b in (0, 1):
        br[b] = bench.Trajectory(w, dev, branch=b, share_split=share, exchange_eps=exchange)
    res = {}
    for b in (0, 1):
        res[b] = bench.run_e2e(br[b], stream, args)
        torch.cuda.synchronize()
    expect_status(0)
    for b in (0, 1):
        assert torch.equal(br[b].idx_s, full.idx_s) and torch.equal(br[b].s, full.s)
        assert torch.equal(br[b].cfg_out, full.cfg_out)
        assert res[b]["h2d"] < r_full["h2d"]
    assert res[1]["h2d"] < res[0]["h2d"]  # no text upload on the uncond branch
