"""safedit_attn_subset_noalloc: the tail-balanced attention with its
workspace in a fixed device array of the library.  Against the entry point
with a caller workspace (safedit_attn_subset_ws) on two calls in a row, and
its refusal of a plan larger than the array.  Collected last, so that it
also runs after every other test has used the device."""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_util import check_attn, expect_status, f64, sd

BF = torch.bfloat16
DEV = "cuda"


def _inputs(B, H, Nq, Nk, D, n_idx, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, n, D, generator=g).to(BF) for n in (Nq, Nk, Nk))
    idx = torch.randperm(Nq, generator=g)[:n_idx].sort().values.to(torch.int32)
    return q.to(DEV), k.to(DEV), v.to(DEV), idx.to(DEV)


@pytest.mark.gpu
def test_noalloc_matches_caller_workspace_on_two_calls_in_a_row():
    # 9 units of 256 rows with 16 key tiles each: the plan splits every unit
    # into 4 key parts (3.6 MB of partial results), so the array is used
    B, H, Nq, Nk, D, n = 1, 3, 2000, 2000, 96, 600
    need = sd().safedit_attn_subset_workspace_size(B, H, n, Nk, D)
    assert 0 < need <= sd().ATTN_NOALLOC_SCRATCH_BYTES
    for call, seed in enumerate((11, 12)):
        q, k, v, idx = _inputs(B, H, Nq, Nk, D, n, seed)
        ws = torch.empty(need, dtype=torch.uint8, device=DEV)
        ref = torch.zeros(B, H, n, D, dtype=BF, device=DEV)
        sd().safedit_attn_subset_ws(q, k, v, idx, n, None, None, 0.0, ref, 0, ws)
        got = torch.zeros_like(ref)
        sd().safedit_attn_subset_noalloc(q, k, v, idx, n, None, None, 0.0, got, 0)
        expect_status(0)
        check_attn(f64(got), f64(ref), f"call {call + 1}")
    # a scattered output through the array: the S rows land at their token
    # index, the other rows of the state are untouched
    state = torch.randn(B, H, Nq, D, generator=torch.Generator().manual_seed(5)).to(BF).to(DEV)
    before = state.clone()
    sd().safedit_attn_subset_noalloc(q, k, v, idx, n, None, None, 0.0, state, 1)
    expect_status(0)
    check_attn(f64(state[:, :, idx.long()]), f64(ref), "scattered")
    keep = torch.ones(Nq, dtype=torch.bool, device=DEV)
    keep[idx.long()] = False
    assert torch.equal(state[:, :, keep], before[:, :, keep])


@pytest.mark.gpu
def test_noalloc_refuses_a_plan_larger_than_its_array():
    # 256 units = 1 wave + 108 over 200 key tiles: 108 units in 4 parts, 43 MB
    B, H, Nq, Nk, D = 1, 8, 8192, 25600, 96
    need = sd().safedit_attn_subset_workspace_size(B, H, Nq, Nk, D)
    assert need > sd().ATTN_NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, H, Nq, D, dtype=BF, device=DEV)
    k = torch.zeros(B, H, Nk, D, dtype=BF, device=DEV)
    out = torch.zeros_like(q)
    n0 = sd().safedit_kernel_launch_count()
    with pytest.raises(sd().SafeditError) as e:
        sd().safedit_attn_subset_noalloc(q, k, k, None, 0, None, None, 0.0, out, 0)
    assert e.value.code == sd().ERR_UNSUPPORTED
    assert sd().safedit_kernel_launch_count() == n0
    expect_status(0)


def test_noalloc_limit_is_checked_on_the_host_before_any_launch():
    """On the host alone: an oversize plan is refused from the shapes (fake
    device pointers, never dereferenced), a missing tensor is an argument
    error, and the small test shape above fits the array."""
    lib = sd()
    T = lib.SafeditTensor

    def desc(shape):
        strides, acc = [], 1
        for n in reversed(shape):
            strides.insert(0, acc)
            acc *= n
        t = T()
        t.data = ctypes.c_void_p(0x100000)
        t.dtype = lib.BF16
        t.ndim = 4
        for i in range(4):
            t.dims[i] = shape[i]
            t.strides[i] = strides[i]
        return t

    f = lib._lib.safedit_attn_subset_noalloc
    q, k = desc((1, 8, 8192, 96)), desc((1, 8, 25600, 96))
    R = ctypes.byref
    assert f(R(q), R(k), R(k), None, 0, None, None, 0.0, R(q), 0, None) == lib.ERR_UNSUPPORTED
    assert f(None, R(k), R(k), None, 0, None, None, 0.0, R(q), 0, None) == lib.ERR_INVALID_ARG
    assert lib.safedit_attn_subset_workspace_size(1, 3, 600, 2000, 96) <= lib.ATTN_NOALLOC_SCRATCH_BYTES
    assert np.isclose(lib.ATTN_NOALLOC_SCRATCH_BYTES, 24 * 2 ** 20)
