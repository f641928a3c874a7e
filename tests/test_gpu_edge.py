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
    # the tail-balanced entry points: no workspace needed, nothing launched
    assert sd().safedit_attn_subset_workspace_size(1, 2, 0, 64, 96) == 0
    _no_launch(lambda: sd().safedit_attn_subset_ws(q, k, k, idx, 0, None, None, 0.0, state, 1, None))
    _no_launch(lambda: sd().safedit_attn_subset_noalloc(q, k, k, idx, 0, None, None, 0.0, state, 1))
    assert torch.equal(state.view(torch.int16), before.view(torch.int16))


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


@pytest.fixture
def index_check():
    prev = sd().safedit_debug_set_index_check(True)
    yield
    sd().safedit_debug_set_index_check(prev)


def test_debug_index_check_flags_duplicates(index_check):
    """Debug mode: every scattering index vector is checked before the
    scatter.  A duplicate (two writers for one row) or an out-of-range entry
    sets SAFEDIT_ERR_INDEX; a unique vector passes and the results are the
    ones the unchecked calls give.  Index ranges wider than one shared-memory
    bitmap window (1.8 M rows) are checked window by window."""
    B, H, N, D, kr = 1, 2, 300, 64, 40
    g = torch.Generator().manual_seed(3)
    uniq = torch.randperm(N, generator=g)[:kr].to(torch.int32).to(DEV)
    dup = uniq.clone()
    dup[17] = dup[3]
    src = torch.randn(B, H, kr, D, generator=g).to(BF).to(DEV)
    dst = torch.zeros(B, H, N, D, dtype=BF, device=DEV)
    q = torch.randn(B, H, N, D, generator=g).to(BF).to(DEV)
    a = torch.randn(kr, 64, generator=g).to(BF).to(DEV)
    w = torch.randn(64, 64, generator=g).to(BF).to(DEV)
    y = torch.zeros(N, 64, dtype=BF, device=DEV)
    calls = [
        lambda ix: sd().safedit_scatter_state([src], [dst], ix, kr),
        lambda ix: sd().safedit_attn_subset(q, q, q, ix, kr, None, None, 0.0, dst, 1),
        lambda ix: sd().safedit_gemm_bias_act(a, w, None, 0, ix, y),
    ]
    for call in calls:
        call(uniq)
        expect_status(0)
        call(dup)
        expect_status(sd().ERR_INDEX)
    # without the check a duplicate goes unnoticed (the caller's contract)
    sd().safedit_debug_set_index_check(False)
    sd().safedit_scatter_state([src], [dst], dup, kr)
    expect_status(0)
    sd().safedit_debug_set_index_check(True)
    # more rows than one bitmap window: a duplicate in the second window
    big = 1_859_584 + 1000
    src2 = torch.randn(1, 1, 3, 8, generator=g).to(BF).to(DEV)
    dst2 = torch.zeros(1, 1, big, 8, dtype=BF, device=DEV)
    ix2 = torch.tensor([5, big - 1, big - 1], dtype=torch.int32, device=DEV)
    sd().safedit_scatter_state([src2], [dst2], ix2, 3)
    expect_status(sd().ERR_INDEX)
    ix2[2] = big - 2
    sd().safedit_scatter_state([src2], [dst2], ix2, 3)
    expect_status(0)
