"""The 2560^2 workload's non-attention rows at full size, in the launch
configurations the benchmark times, against the oracle on sampled outputs:
cross-attention probabilities of the cond branch, their aggregation, the
fused PCSP score, the split, the K/V state scatter and the guidance combine.
(The attention launches of this workload have their own full-size tests.)"""
import numpy as np
import pytest
import torch

import oracle
from spatially_adaptive_dit_b200 import workloads as wl
from tests.gpu_util import CFG_REL, XATTN_MAX_ABS, expect_status, sd

pytestmark = pytest.mark.gpu
DEV = "cuda"
W = wl.W2560


@pytest.fixture(scope="module")
def pcsp():
    """The warm-up step's probabilities, unfused aggregation and fused score."""
    q_img, k_txt, valid, content = wl.text(W, device=DEV)
    P = torch.full((W.H, W.N, W.L), -1.0, device=DEV)
    sd().safedit_cross_attn_probs(q_img, k_txt, valid, 0, 0.0, P)
    score = torch.zeros(W.N, dtype=torch.float64, device=DEV)
    sd().safedit_partition_accumulate(P, content, score)
    fused = torch.zeros(W.N, dtype=torch.float64, device=DEV)
    sd().safedit_pcsp_score(q_img, k_txt, valid, content, 0, 0.0, fused)
    expect_status(0)
    return dict(q_img=q_img, k_txt=k_txt, valid=valid, content=content, P=P, score=score, fused=fused)


def test_probabilities_sampled_rows(pcsp):
    rows = torch.as_tensor(np.linspace(0, W.N - 1, 96).astype(np.int64), device=DEV)
    valid = pcsp["valid"][0].cpu().numpy()
    for h in (0, 11, 23):
        ref = oracle.cross_attn_probs(pcsp["q_img"][0, h:h + 1, rows].double().cpu(),
                                      pcsp["k_txt"][0, h:h + 1].double().cpu(), valid)
        got = pcsp["P"][h:h + 1, rows].double().cpu().numpy()
        assert np.abs(got - ref).max() <= XATTN_MAX_ABS
        assert np.all(got[..., valid == 0] == 0.0)


def test_aggregation_sampled_rows_and_fused_score(pcsp):
    """The unfused aggregation against the oracle on the GPU's own P (the same
    probabilities on both sides: 1e-12); the fused score, which never writes
    P, against the oracle's fp64 probabilities (r24: 1e-5 of the largest)."""
    rows = np.linspace(0, W.N - 1, 256).astype(np.int64)
    rt = torch.as_tensor(rows, device=DEV)
    content = pcsp["content"].cpu().numpy()
    ref_gpu_p = oracle.partition_accumulate(pcsp["P"][:, rt].double().cpu(), content)
    got = pcsp["score"][rt].cpu().numpy()
    assert np.abs(got - ref_gpu_p).max() <= 1e-12 * np.abs(ref_gpu_p).max()
    valid = pcsp["valid"][0].cpu().numpy()
    Pr = oracle.cross_attn_probs(pcsp["q_img"][0, :, rt].double().cpu(), pcsp["k_txt"][0].double().cpu(), valid)
    ref = oracle.partition_accumulate(Pr, content)
    for s in (pcsp["fused"], pcsp["score"]):
        assert np.abs(s[rt].cpu().numpy() - ref).max() <= 1e-5 * np.abs(ref).max()


def test_split_of_the_fused_score(pcsp):
    """The split the trajectory makes from the fused score: bit-exact against
    the oracle's selection on the same score vector."""
    idx_s = torch.empty(W.k, dtype=torch.int32, device=DEV)
    idx_c = torch.empty(W.N - W.k, dtype=torch.int32, device=DEV)
    s = torch.empty(W.N, device=DEV)
    sd().safedit_partition_finalize(pcsp["fused"], W.N, W.k, idx_s, idx_c, s)
    expect_status(0)
    r_s, r_c, r_sv = oracle.partition_select(pcsp["fused"].cpu().numpy(), W.k)
    assert np.array_equal(idx_s.cpu().numpy(), r_s)
    assert np.array_equal(idx_c.cpu().numpy(), r_c)
    assert np.array_equal(s.cpu().numpy(), r_sv)


def test_state_scatter_and_guidance_combine(pcsp):
    """K_S and V_S scattered into the 236 MB states in one launch: bit-exact
    on sampled slices (every S row replaced, every C row untouched); the
    guidance combine of the full [N, F] prediction."""
    idx_s = torch.empty(W.k, dtype=torch.int32, device=DEV)
    s = torch.empty(W.N, device=DEV)
    sd().safedit_partition_finalize(pcsp["fused"], W.N, W.k, idx_s, None, s)
    _, k_full, v_full = wl.qkv(W, device=DEV)
    k_s, v_s = wl.fresh_sensitive_kv(W, W.k, step=1, device=DEV)
    k_state, v_state = k_full.clone(), v_full.clone()
    sd().safedit_scatter_state([k_s, v_s], [k_state, v_state], idx_s, W.k)
    expect_status(0)
    ix = idx_s.cpu().numpy()
    for src, before, after in ((k_s, k_full, k_state), (v_s, v_full, v_state)):
        for (b, h) in ((0, 0), (1, 23), (0, 17)):
            ref = oracle.scatter_rows(src[b, h].view(torch.int16).cpu().numpy(),
                                      before[b, h].view(torch.int16).cpu().numpy(), ix)
            assert np.array_equal(after[b, h].view(torch.int16).cpu().numpy(), ref)
    eps_c, eps_u = wl.cfg_preds(W, device=DEV)
    out = torch.empty_like(eps_c)
    sd().safedit_sw_cfg(eps_c, eps_u, s, W.gamma_ctx, W.gamma_sens, out)
    expect_status(0)
    c, u = eps_c.double().cpu().numpy(), eps_u.double().cpu().numpy()
    ref = oracle.sw_cfg(c, u, s.cpu().numpy(), W.gamma_ctx, W.gamma_sens)
    g = np.abs(c - u) * max(W.gamma_ctx, W.gamma_sens) + np.abs(u)
    assert np.all(np.abs(out.double().cpu().numpy() - ref) <= CFG_REL * g + 1e-30)
