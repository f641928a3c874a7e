"""Fused PCSP score (cross-attention probabilities aggregated without
materialising P) against the oracle's C1 + C2 composition, against the
unfused GPU path, and for determinism."""
import numpy as np
import pytest
import torch

import oracle
from spatially_adaptive_dit_b200 import workloads as wl
from tests.gpu_util import expect_status, f64, sd

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _oracle_score(q_img, k_txt, valid, content, b):
    P = oracle.cross_attn_probs(f64(q_img[b]), f64(k_txt[b]), valid[b].cpu().numpy())
    return oracle.partition_accumulate(P, content.cpu().numpy())


def _fused(q_img, k_txt, valid, content, b, start=None):
    N = q_img.shape[2]
    score = torch.zeros(N, dtype=torch.float64, device=DEV) if start is None else start.clone()
    sd().safedit_pcsp_score(q_img, k_txt, valid, content, b, 0.0, score)
    expect_status(0)
    return score


@pytest.mark.parametrize("w", [wl.TINY, wl.W1024])
def test_fused_score_matches_oracle_and_split(w):
    q_img, k_txt, valid, content = wl.text(w, device=DEV)
    score = _fused(q_img, k_txt, valid, content, 0).cpu().numpy()
    ref = _oracle_score(q_img, k_txt, valid, content, 0)
    assert np.abs(score - ref).max() <= 1e-5 * np.abs(ref).max()
    k = w.k
    idx = torch.empty(k, dtype=torch.int32, device=DEV)
    sd().safedit_partition_finalize(torch.tensor(score, device=DEV), w.N, k, idx, None, None)
    r_s, _, _ = oracle.partition_select(ref, k)
    tau = np.sort(ref)[::-1][k - 1]
    near = set(np.nonzero(np.abs(ref - tau) <= 1e-6 * abs(tau))[0].tolist())
    assert set(idx.cpu().numpy().tolist()) - near == set(r_s.tolist()) - near


@pytest.mark.parametrize("B,H,N,L,D,b", [(2, 3, 300, 40, 128, 1), (1, 1, 129, 256, 96, 0),
                                          (1, 2, 64, 17, 64, 0)])
def test_fused_score_ragged_shapes_and_accumulation(B, H, N, L, D, b):
    g = torch.Generator().manual_seed(N * 7 + L)
    q_img = torch.randn(B, H, N, D, generator=g).to(torch.bfloat16).to(DEV)
    k_txt = torch.randn(B, H, L, D, generator=g).to(torch.bfloat16).to(DEV)
    valid = (torch.rand(B, L, generator=g) < 0.6).to(torch.uint8)
    valid[:, 0] = 1
    content = (torch.rand(L, generator=g) < 0.7).to(torch.uint8)
    valid, content = valid.to(DEV), content.to(DEV)
    start = torch.rand(N, dtype=torch.float64, generator=g).to(DEV)
    score = _fused(q_img, k_txt, valid, content, b, start).cpu().numpy()
    ref = start.cpu().numpy() + _oracle_score(q_img, k_txt, valid, content, b)
    assert np.abs(score - ref).max() <= 1e-5 * np.abs(ref).max()


def test_fused_equals_unfused_gpu_path_and_is_deterministic():
    w = wl.W1024
    q_img, k_txt, valid, content = wl.text(w, device=DEV)
    fused = _fused(q_img, k_txt, valid, content, 0)
    again = _fused(q_img, k_txt, valid, content, 0)
    assert torch.equal(fused, again)
    P = torch.empty(w.H, w.N, w.L, device=DEV)
    sd().safedit_cross_attn_probs(q_img, k_txt, valid, 0, 0.0, P)
    unfused = torch.zeros(w.N, dtype=torch.float64, device=DEV)
    sd().safedit_partition_accumulate(P, content, unfused)
    expect_status(0)
    assert (fused - unfused).abs().max().item() <= 1e-5 * unfused.abs().max().item()
