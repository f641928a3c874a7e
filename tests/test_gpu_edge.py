"""Empty and degenerate inputs through the C ABI: every entry point accepts
work of size zero (null data pointers of empty tensors included), launches
nothing and leaves its outputs untouched."""
import pytest
import torch

from tests.gpu_util import expect_status, sd

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF = torch.bfloat16


def _no_launch(fn):
    n0 = sd().safedit_kernel_launch_count()
    fn()
    torch.cuda.synchronize()
    assert sd().safedit_kernel_launch_count() == n0
    expect_status(0)


def test_attention_without_rows():
    q = torch.randn(1, 2, 64, 96, device=DEV).to(BF)
    k = torch.randn(1, 2, 64, 96, device=DEV).to(BF)
    idx = torch.empty(0, dtype=torch.int32, device=DEV)
    out = torch.empty(1, 2, 0, 96, dtype=BF, device=DEV)
    _no_launch(lambda: sd().safedit_attn_subset(q, k, k, idx, 0, None, None, 0.0, out, 0))
    # scattered output: the state keeps every byte
    state = torch.randn(1, 2, 64, 96, device=DEV).to(BF)
    before = state.clone()
    _no_launch(lambda: sd().safedit_attn_subset(q, k, k, idx, 0, None, None, 0.0, state, 1))
    assert torch.equal(state.view(torch.int16), before.view(torch.int16))
    # no query rows at all
    q0 = torch.empty(1, 2, 0, 96, dtype=BF, device=DEV)
    _no_launch(lambda: sd().safedit_attn_subset(q0, k, k, None, 0, None, None, 0.0, out, 0))


def test_row_copies_without_rows():
    dst = torch.randn(2, 3, 50, 64, device=DEV).to(BF)
    before = dst.clone()
    src = torch.empty(2, 3, 0, 64, dtype=BF, device=DEV)
    idx = torch.empty(0, dtype=torch.int32, device=DEV)
    _no_launch(lambda: sd().safedit_scatter_state([src], [dst], idx, 0))
    _no_launch(lambda: sd().safedit_gather_rows([dst], [src], idx, 0))
    assert torch.equal(dst.view(torch.int16), before.view(torch.int16))


def test_guidance_without_tokens():
    e = torch.empty(0, 16, device=DEV)
    s = torch.empty(0, device=DEV)
    _no_launch(lambda: sd().safedit_sw_cfg(e, e, s, 3.0, 5.0, e))
    _no_launch(lambda: sd().safedit_stepcache_sw_cfg(e, e, e, e, s, 0.5, 3.0, 5.0, e))


def test_partition_without_tokens():
    q_img = torch.empty(1, 2, 0, 64, dtype=BF, device=DEV)
    k_txt = torch.randn(1, 2, 32, 64, device=DEV).to(BF)
    valid = torch.ones(1, 32, dtype=torch.uint8, device=DEV)
    content = torch.ones(32, dtype=torch.uint8, device=DEV)
    P = torch.empty(2, 0, 32, device=DEV)
    score = torch.empty(0, dtype=torch.float64, device=DEV)
    _no_launch(lambda: sd().safedit_cross_attn_probs(q_img, k_txt, valid, 0, 0.0, P))
    _no_launch(lambda: sd().safedit_partition_accumulate(P, content, score))
    _no_launch(lambda: sd().safedit_pcsp_score(q_img, k_txt, valid, content, 0, 0.0, score))
    _no_launch(lambda: sd().safedit_partition_finalize(score, 0, 0, None, None, None))


def test_projection_without_rows_or_columns():
    a = torch.empty(0, 64, dtype=BF, device=DEV)
    w = torch.randn(64, 64, device=DEV).to(BF)
    out = torch.empty(0, 64, dtype=BF, device=DEV)
    _no_launch(lambda: sd().safedit_gemm_bias_act(a, w, None, 1, None, out))
    a1 = torch.randn(5, 64, device=DEV).to(BF)
    w0 = torch.empty(0, 64, dtype=BF, device=DEV)
    out0 = torch.empty(5, 0, dtype=BF, device=DEV)
    _no_launch(lambda: sd().safedit_gemm_bias_act(a1, w0, None, 0, None, out0))
