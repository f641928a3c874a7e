"""Failure detection without a GPU fault: with the debug wait limit at 0 the
pipelined kernels' bounded waits give up at once; each CTA then raises its
abort flag, drains its in-flight TMA loads and MMAs, frees TMEM and returns,
and the status word reports SAFEDIT_ERR_TIMEOUT.  The context must stay
usable: the next call with the normal limit reproduces the reference output
bit for bit."""
import pytest
import torch

from tests.gpu_util import expect_status, sd

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _attn_case():
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 4, 1024, 96, generator=g).to(torch.bfloat16).to(DEV)
    k = torch.randn(1, 4, 1024, 96, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(1, 4, 1024, 96, generator=g).to(torch.bfloat16).to(DEV)
    idx = torch.arange(0, 1024, 3, dtype=torch.int32, device=DEV)
    return q, k, v, idx


def _run_attn(q, k, v, idx):
    out = torch.zeros(1, 4, idx.numel(), 96, dtype=torch.bfloat16, device=DEV)
    sd().safedit_attn_subset(q, k, v, idx, idx.numel(), None, None, 0.0, out, 0)
    return out


def _run_xattn():
    g = torch.Generator().manual_seed(6)
    qi = torch.randn(1, 4, 2048, 96, generator=g).to(torch.bfloat16).to(DEV)
    kt = torch.randn(1, 4, 256, 96, generator=g).to(torch.bfloat16).to(DEV)
    valid = torch.ones(1, 256, dtype=torch.uint8, device=DEV)
    P = torch.zeros(4, 2048, 256, device=DEV)
    sd().safedit_cross_attn_probs(qi, kt, valid, 0, 0.0, P)
    return P


def _run_pcsp():
    g = torch.Generator().manual_seed(9)
    qi = torch.randn(1, 4, 2048, 96, generator=g).to(torch.bfloat16).to(DEV)
    kt = torch.randn(1, 4, 256, 96, generator=g).to(torch.bfloat16).to(DEV)
    valid = torch.ones(1, 256, dtype=torch.uint8, device=DEV)
    content = torch.zeros(256, dtype=torch.uint8, device=DEV)
    content[1:200] = 1
    score = torch.zeros(2048, dtype=torch.float64, device=DEV)
    sd().safedit_pcsp_score(qi, kt, valid, content, 0, 0.0, score)
    return score


def _run_gemm():
    g = torch.Generator().manual_seed(7)
    a = torch.randn(1000, 512, generator=g).to(torch.bfloat16).to(DEV)
    w = torch.randn(768, 512, generator=g).to(torch.bfloat16).to(DEV)
    out = torch.zeros(1000, 768, dtype=torch.bfloat16, device=DEV)
    sd().safedit_gemm_bias_act(a, w, None, 1, None, out)
    return out


def test_bounded_wait_timeout_is_reported_and_context_survives():
    q, k, v, idx = _attn_case()
    ref = _run_attn(q, k, v, idx)
    ref_p = _run_xattn()
    ref_g = _run_gemm()
    ref_s = _run_pcsp()
    expect_status(0)
    old = sd().safedit_debug_set_wait_limit_ns(0)
    try:
        _run_attn(q, k, v, idx)
        expect_status(sd().ERR_TIMEOUT)
        _run_xattn()
        expect_status(sd().ERR_TIMEOUT)
        _run_gemm()
        expect_status(sd().ERR_TIMEOUT)
        _run_pcsp()
        expect_status(sd().ERR_TIMEOUT)
    finally:
        sd().safedit_debug_set_wait_limit_ns(old)
    again = _run_attn(q, k, v, idx)
    again_p = _run_xattn()
    again_g = _run_gemm()
    again_s = _run_pcsp()
    expect_status(0)
    assert torch.equal(again, ref)
    assert torch.equal(again_p, ref_p)
    assert torch.equal(again_g, ref_g)
    assert torch.equal(again_s, ref_s)


def test_tail_split_timeout_is_reported_and_context_survives():
    """The tail-balanced launch (whole units, key-range parts that may overlap
    them, the merge) with the wait limit at 0: every CTA of both attention
    launches gives up, the part launch still completes after the whole-unit
    one, the status word reports SAFEDIT_ERR_TIMEOUT, and the next call
    reproduces the reference bit for bit."""
    g = torch.Generator().manual_seed(8)
    q, k, v = (torch.randn(1, 50, 2000, 96, generator=g).to(torch.bfloat16).to(DEV) for _ in range(3))
    idx = torch.arange(0, 2000, 3, dtype=torch.int32, device=DEV)[:600]
    nb = sd().safedit_attn_subset_workspace_size(1, 50, 600, 2000, 96)
    assert nb > 0  # 150 units: 148 whole, 2 in key parts
    ws = torch.empty(nb, dtype=torch.uint8, device=DEV)

    def run():
        out = torch.zeros(1, 50, 600, 96, dtype=torch.bfloat16, device=DEV)
        sd().safedit_attn_subset_ws(q, k, v, idx, 600, None, None, 0.0, out, 0, ws)
        return out

    ref = run()
    expect_status(0)
    old = sd().safedit_debug_set_wait_limit_ns(0)
    try:
        run()
        expect_status(sd().ERR_TIMEOUT)
    finally:
        sd().safedit_debug_set_wait_limit_ns(old)
    again = run()
    expect_status(0)
    assert torch.equal(again, ref)


def test_device_errors_do_not_poison_later_calls():
    q, k, v, idx = _attn_case()
    ref = _run_attn(q, k, v, idx)
    bad = idx.clone()
    bad[0] = 10 ** 6
    _run_attn(q, k, v, bad)
    expect_status(sd().ERR_INDEX)
    assert torch.equal(_run_attn(q, k, v, idx), ref)
    expect_status(0)
