"""CPU-side checks of the C-ABI library: it loads, exports every entry point
include/safedit.h declares, and rejects bad arguments on the host before any
CUDA call (no GPU needed, nothing is launched)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sd():
    from spatially_adaptive_dit_b200 import build
    build.build()
    from spatially_adaptive_dit_b200 import safedit
    return safedit


def _declared():
    with open(os.path.join(ROOT, "include", "safedit.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(safedit_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(sd):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(sd.lib(), n), n
        assert hasattr(sd, n), f"python binding lacks {n}"
    assert set(names) == set(sd.EXPORTED)


def test_status_strings_and_counters(sd):
    assert sd.status_string(0) == "ok"
    for c in range(1, 10):
        assert sd.status_string(c) not in ("ok", "unknown status")
    assert sd.status_string(77) == "unknown status"
    assert sd.safedit_kernel_launch_count() >= 0
    old = sd.safedit_debug_set_wait_limit_ns(12345)
    assert sd.safedit_debug_set_wait_limit_ns(old) == 12345
    prev = sd.safedit_debug_set_index_check(True)
    assert sd.safedit_debug_set_index_check(prev) is True


def test_sw_cfg_argument_checks(sd):
    """Prediction dtypes: both f32 or both bf16; the output is f32."""
    n, f = 64, 16
    c32 = _desc(sd, (n, f), (f, 1), sd.F32)
    c16 = _desc(sd, (n, f), (f, 1), sd.BF16)
    out = _desc(sd, (n, f), (f, 1), sd.F32)
    out16 = _desc(sd, (n, f), (f, 1), sd.BF16)
    call = lambda c, u, o: sd.raw_call("safedit_sw_cfg", ctypes.byref(c), ctypes.byref(u), ctypes.c_void_p(0x20000),
                                       ctypes.c_float(3.0), ctypes.c_float(5.0), ctypes.byref(o), None)
    assert call(c32, c16, out) == sd.ERR_DTYPE
    assert call(c16, c32, out) == sd.ERR_DTYPE
    assert call(c16, c16, out16) == sd.ERR_DTYPE
    wide = _desc(sd, (n, f), (f, 2), sd.BF16)
    assert call(wide, c16, out) == sd.ERR_ALIGNMENT


def _desc(sd, dims, strides, dtype, ptr=0x10000):
    d = sd.SafeditTensor()
    d.data = ptr
    d.dtype = dtype
    d.ndim = len(dims)
    for i, (a, b) in enumerate(zip(dims, strides)):
        d.dims[i] = a
        d.strides[i] = b
    return d


def _bhnd(sd, B, H, N, D, dtype=None, ptr=0x10000, strides=None):
    dtype = sd.BF16 if dtype is None else dtype
    st = strides or (H * N * D, N * D, D, 1)
    return _desc(sd, (B, H, N, D), st, dtype, ptr)


def test_attn_host_validation(sd):
    call = lambda *a: sd.raw_call("safedit_attn_subset", *a)  # noqa: E731
    q, k, v, o = (_bhnd(sd, 1, 2, 256, 64) for _ in range(4))
    R = ctypes.byref
    # null tensor
    assert call(None, R(k), R(v), None, 0, None, None, 0.0, R(o), 0, None) == sd.ERR_INVALID_ARG
    # wrong dtype
    qf = _bhnd(sd, 1, 2, 256, 64, dtype=sd.F32)
    assert call(R(qf), R(k), R(v), None, 0, None, None, 0.0, R(o), 0, None) == sd.ERR_DTYPE
    # unsupported head dim
    q80, k80, v80, o80 = (_bhnd(sd, 1, 2, 256, 80) for _ in range(4))
    assert call(R(q80), R(k80), R(v80), None, 0, None, None, 0.0, R(o80), 0, None) == sd.ERR_UNSUPPORTED
    # misaligned pointer / stride
    qm = _bhnd(sd, 1, 2, 256, 64, ptr=0x10008)
    assert call(R(qm), R(k), R(v), None, 0, None, None, 0.0, R(o), 0, None) == sd.ERR_ALIGNMENT
    qs = _bhnd(sd, 1, 2, 256, 64, strides=(2 * 256 * 68, 256 * 68, 68, 1))
    assert call(R(qs), R(k), R(v), None, 0, None, None, 0.0, R(o), 0, None) == sd.ERR_ALIGNMENT
    # shape mismatch between k and v
    v2 = _bhnd(sd, 1, 2, 128, 64)
    assert call(R(q), R(k), R(v2), None, 0, None, None, 0.0, R(o), 0, None) == sd.ERR_SHAPE
    # compact output must have n_idx rows
    o_bad = _bhnd(sd, 1, 2, 10, 64)
    assert call(R(q), R(k), R(v), ctypes.c_void_p(0x20000), 11, None, None, 0.0, R(o_bad), 0,
                None) == sd.ERR_SHAPE
    assert call(R(q), R(k), R(v), None, 0, None, None, 0.0, R(o), 2, None) == sd.ERR_INVALID_ARG
    # key pad of the wrong length, bias of the wrong dtype
    pad = _desc(sd, (1, 255), (256, 1), sd.F32)
    assert call(R(q), R(k), R(v), None, 0, R(pad), None, 0.0, R(o), 0, None) == sd.ERR_SHAPE
    bias = _desc(sd, (1, 1, 256, 256), (65536, 65536, 256, 1), sd.F16)
    assert call(R(q), R(k), R(v), None, 0, None, R(bias), 0.0, R(o), 0, None) == sd.ERR_DTYPE
    # key pad: batch stride not a 16-byte multiple, inner stride not 1, misaligned data
    for strides, ptr in (((258, 1), 0x1000), ((512, 2), 0x1000), ((256, 1), 0x1008)):
        padb = _desc(sd, (1, 256), strides, sd.F32, ptr=ptr)
        assert call(R(q), R(k), R(v), None, 0, R(padb), None, 0.0, R(o), 0, None) == sd.ERR_ALIGNMENT
    # bias: a bf16 row stride that is not a multiple of 8 elements (an f32 one
    # of 4 would pass), a head dim that is neither 1 nor H, a row count not Nq
    bias_s = _desc(sd, (1, 1, 256, 256), (260 * 256, 260 * 256, 260, 1), sd.BF16)
    assert call(R(q), R(k), R(v), None, 0, None, R(bias_s), 0.0, R(o), 0, None) == sd.ERR_ALIGNMENT
    bias_h = _desc(sd, (1, 3, 256, 256), (3 * 65536, 65536, 256, 1), sd.BF16)
    assert call(R(q), R(k), R(v), None, 0, None, R(bias_h), 0.0, R(o), 0, None) == sd.ERR_SHAPE
    bias_r = _desc(sd, (1, 1, 200, 256), (51200, 51200, 256, 1), sd.F32)
    assert call(R(q), R(k), R(v), None, 0, None, R(bias_r), 0.0, R(o), 0, None) == sd.ERR_SHAPE


def test_bandwidth_kernels_host_validation(sd):
    R = ctypes.byref
    src = (sd.SafeditTensor * 1)(_bhnd(sd, 1, 2, 10, 96))
    dst = (sd.SafeditTensor * 1)(_bhnd(sd, 1, 2, 100, 96))
    f = lambda *a: sd.raw_call("safedit_scatter_state", *a)  # noqa: E731
    assert f(src, dst, 0, ctypes.c_void_p(0x20000), 10, None) == sd.ERR_INVALID_ARG
    assert f(src, dst, 5, ctypes.c_void_p(0x20000), 10, None) == sd.ERR_INVALID_ARG
    assert f(src, dst, 1, None, 10, None) == sd.ERR_INVALID_ARG
    assert f(src, dst, 1, ctypes.c_void_p(0x20000), 11, None) == sd.ERR_SHAPE
    dst_f = (sd.SafeditTensor * 1)(_bhnd(sd, 1, 2, 100, 96, dtype=sd.F32))
    assert f(src, dst_f, 1, ctypes.c_void_p(0x20000), 10, None) == sd.ERR_DTYPE
    # rows of 6 bf16 are not 16-byte multiples
    src6 = (sd.SafeditTensor * 1)(_bhnd(sd, 1, 2, 10, 6))
    dst6 = (sd.SafeditTensor * 1)(_bhnd(sd, 1, 2, 100, 6))
    assert f(src6, dst6, 1, ctypes.c_void_p(0x20000), 10, None) == sd.ERR_ALIGNMENT

    c = _desc(sd, (100, 16), (16, 1), sd.F32)
    u = _desc(sd, (100, 16), (16, 1), sd.F32)
    o_bad = _desc(sd, (100, 8), (8, 1), sd.F32)
    g = lambda *a: sd.raw_call("safedit_sw_cfg", *a)  # noqa: E731
    assert g(R(c), R(u), None, 3.0, 5.0, R(u), None) == sd.ERR_INVALID_ARG
    assert g(R(c), R(u), ctypes.c_void_p(0x30000), 3.0, 5.0, R(o_bad), None) == sd.ERR_SHAPE
    cb = _desc(sd, (100, 16), (16, 1), sd.BF16)
    assert g(R(cb), R(u), ctypes.c_void_p(0x30000), 3.0, 5.0, R(u), None) == sd.ERR_DTYPE

    fin = lambda *a: sd.raw_call("safedit_partition_finalize", *a)  # noqa: E731
    assert fin(None, 10, 3, None, None, None, None) == sd.ERR_INVALID_ARG
    assert fin(ctypes.c_void_p(0x40000), 10, 11, None, None, None, None) == sd.ERR_INVALID_ARG
    assert fin(ctypes.c_void_p(0x40000), 10, -1, None, None, None, None) == sd.ERR_INVALID_ARG

    P = _desc(sd, (2, 16, 32), (512, 32, 1), sd.F16)  # P in f32 or bf16 only
    acc = lambda *a: sd.raw_call("safedit_partition_accumulate", *a)  # noqa: E731
    assert acc(R(P), ctypes.c_void_p(0x50000), ctypes.c_void_p(0x60000), None) == sd.ERR_DTYPE
    Pf = _desc(sd, (2, 16, 32), (512, 32, 2), sd.F32)
    assert acc(R(Pf), ctypes.c_void_p(0x50000), ctypes.c_void_p(0x60000), None) == sd.ERR_ALIGNMENT

    m = _desc(sd, (4, 4, 8, 8), (256, 64, 8, 1), sd.I32)
    mk = lambda *a: sd.raw_call("safedit_mask_is_row_constant", *a)  # noqa: E731
    assert mk(R(m), ctypes.c_void_p(0x70000), None, None) == sd.ERR_DTYPE
    m1 = _desc(sd, (8,), (1,), sd.F32)
    assert mk(R(m1), ctypes.c_void_p(0x70000), None, None) == sd.ERR_SHAPE
    m2 = _desc(sd, (8, 8), (8, 2), sd.F32)
    assert mk(R(m2), ctypes.c_void_p(0x70000), None, None) == sd.ERR_ALIGNMENT

    xq = _bhnd(sd, 2, 2, 256, 64)
    xk = _bhnd(sd, 2, 2, 300, 64)
    xp = _desc(sd, (2, 256, 300), (256 * 300, 300, 1), sd.F32)
    x = lambda *a: sd.raw_call("safedit_cross_attn_probs", *a)  # noqa: E731
    assert x(R(xq), R(xk), ctypes.c_void_p(0x80000), 0, 0.0, R(xp), None) == sd.ERR_UNSUPPORTED
    xk2 = _bhnd(sd, 2, 2, 32, 64)
    xp2 = _desc(sd, (2, 256, 32), (256 * 32, 32, 1), sd.F32)
    assert x(R(xq), R(xk2), ctypes.c_void_p(0x80000), 2, 0.0, R(xp2), None) == sd.ERR_INVALID_ARG
    assert x(R(xq), R(xk2), None, 0, 0.0, R(xp2), None) == sd.ERR_INVALID_ARG
    xp3 = _desc(sd, (2, 256, 30), (256 * 30, 30, 1), sd.F32)
    xk3 = _bhnd(sd, 2, 2, 30, 64)
    assert x(R(xq), R(xk3), ctypes.c_void_p(0x80000), 0, 0.0, R(xp3), None) == sd.ERR_ALIGNMENT


def test_attention_tail_split_plan(sd):
    """Workspace the tail-balanced attention needs (148 SMs): the units that do
    not fill the last wave are split over the keys into the s in 2..4 that
    ends the call soonest by the per-CTA cost model (11.6 us + 1.83 us per key
    tile at d = 96), when that saves 3% of the whole launch; each split unit
    keeps s x 256 rows of (d + 2) f32."""
    ws = sd.safedit_attn_subset_workspace_size
    row = lambda d: 256 * (d + 2) * 4
    # 2560^2 SRSU: 30 x 48 = 1440 units = 9 waves + 108; 108 units x 4 parts
    # (3 rounds of 1/4) would save 61 us of 10 rounds x 378 us: under 3%
    assert ws(2, 24, 7680, 25600, 96) == 0
    # 2560^2 anchor: 100 x 48 = 4800 = 32 waves + 64; 64 x 2 saves 1.4%
    assert ws(2, 24, 25600, 25600, 96) == 0
    # 1024^2 SRSU: 5 x 48 = 240 = 1 wave + 92 units of 32 key tiles: two
    # rounds of 1/3 + the merge (70 us) do not beat one whole round (70 us)
    assert ws(2, 24, 1229, 4096, 96) == 0
    # 1024^2 anchor: 16 x 48 = 768 = 5 waves + 28 -> 28 x 4 (one round of 1/4)
    assert ws(2, 24, 4096, 4096, 96) == 28 * 4 * row(96)
    # stress SRSU (with kept masks or not: the same plan): 20 x 32 = 640 =
    # 4 waves + 48 -> 48 x 3 (one round of 1/3)
    assert ws(1, 32, 4915, 16384, 128) == 48 * 3 * row(128)
    # no tail, or too few key tiles to split: nothing
    assert ws(1, 148, 256, 25600, 96) == 0
    assert ws(1, 2, 64, 256, 64) == 0
    assert ws(0, 2, 64, 256, 64) == 0 and ws(1, 2, 64, 4096, 80) == 0
