"""GPU vs oracle parity of the PCSP cross-attention probability producer."""
import numpy as np
import pytest
import torch

import oracle
from spatially_adaptive_dit_b200 import workloads as wl
from tests.gpu_util import XATTN_MAX_ABS, expect_status, f64, sd

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(q_img, k_txt, valid, b, scale=0.0):
    B, H, N, D = q_img.shape
    L = k_txt.shape[2]
    P = torch.full((H, N, L), -1.0, device=DEV)
    sd().safedit_cross_attn_probs(q_img, k_txt, valid, b, scale, P)
    expect_status(0)
    return P


def _check(P, q_img, k_txt, valid, b, heads):
    for h in heads:
        ref = oracle.cross_attn_probs(f64(q_img[b, h:h + 1]), f64(k_txt[b, h:h + 1]),
                                      valid[b].cpu().numpy())
        got = P[h:h + 1].cpu().double().numpy()
        assert np.abs(got - ref).max() <= XATTN_MAX_ABS
        inval = valid[b].cpu().numpy() == 0
        assert np.all(got[..., inval] == 0.0)


def test_tiny_config():
    w = wl.TINY
    q_img, k_txt, valid, _ = wl.text(w)
    P = _run(q_img.to(DEV), k_txt.to(DEV), valid.to(DEV), 0)
    _check(P, q_img, k_txt, valid, 0, range(w.H))


def test_1024_config_cond_branch():
    w = wl.W1024
    q_img, k_txt, valid, _ = wl.text(w, device=DEV)
    P = _run(q_img, k_txt, valid, 0)
    _check(P, q_img, k_txt, valid, 0, [0, 13, 23])
    assert torch.allclose(P.sum(-1), torch.ones_like(P[..., 0]), atol=1e-5)


@pytest.mark.parametrize("N,L,D,b", [(200, 40, 128, 1), (130, 256, 96, 0), (64, 17, 64, 0)])
def test_ragged_and_non_prefix_validity(N, L, D, b):
    g = torch.Generator().manual_seed(N + L)
    q_img = torch.randn(2, 3, N, D, generator=g).to(torch.bfloat16)
    k_txt = torch.randn(2, 3, L, D, generator=g).to(torch.bfloat16)
    valid = (torch.rand(2, L, generator=g) < 0.6).to(torch.uint8)
    valid[:, 0] = 1
    Lp = (L + 3) // 4 * 4
    P_full = torch.full((3, N, Lp), -1.0, device=DEV)
    P = P_full[:, :, :L]
    sd().safedit_cross_attn_probs(q_img.to(DEV), k_txt.to(DEV), valid.to(DEV), b, 0.0, P)
    expect_status(0)
    _check(P, q_img, k_txt, valid, b, range(3))
    if Lp > L:
        assert torch.all(P_full[:, :, L:] == -1.0)  # padding columns of the buffer untouched
