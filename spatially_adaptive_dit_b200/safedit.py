"""Thin ctypes binding of libsafedit.so (include/safedit.h).

Argument marshalling only: torch tensors (device memory allocated by torch)
become `safedit_tensor` descriptors, streams become cudaStream_t handles, and
every non-OK status raises SafeditError.  All computation happens in the
library's CUDA kernels.  Importing this module fails loudly if the library
has not been built: there is no CPU fallback.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsafedit.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m spatially_adaptive_dit_b200.build` "
        "(or __graft_entry__.build()); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)

# ---- enums (mirror include/safedit.h) -------------------------------------
OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_DTYPE, ERR_ALIGNMENT, ERR_INDEX, ERR_UNSUPPORTED, ERR_CUDA, \
    ERR_TIMEOUT, ERR_MASKED_ROW = range(10)
F32, BF16, F16, BOOL, I32, F64, U8 = range(7)

_DTYPE = {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16, torch.bool: BOOL,
          torch.int32: I32, torch.float64: F64, torch.uint8: U8}

EXPORTED = ("safedit_cross_attn_probs", "safedit_partition_accumulate", "safedit_pcsp_score",
            "safedit_partition_finalize", "safedit_mask_is_row_constant", "safedit_attn_subset",
            "safedit_attn_subset_ws", "safedit_attn_subset_workspace_size", "safedit_attn_subset_noalloc",
            "safedit_scatter_state", "safedit_gather_rows", "safedit_sw_cfg", "safedit_stepcache_sw_cfg",
            "safedit_gemm_bias_act", "safedit_get_device_status", "safedit_status_string", "safedit_kernel_launch_count",
            "safedit_debug_set_wait_limit_ns", "safedit_debug_set_index_check")


class SafeditTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("dims", ctypes.c_int64 * 4), ("strides", ctypes.c_int64 * 4)]


class SafeditError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


_T = ctypes.POINTER(SafeditTensor)
_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_f32 = ctypes.c_float

_lib.safedit_cross_attn_probs.argtypes = [_T, _T, _vp, _i32, _f32, _T, _vp]
_lib.safedit_partition_accumulate.argtypes = [_T, _vp, _vp, _vp]
_lib.safedit_partition_finalize.argtypes = [_vp, _i32, _i32, _vp, _vp, _vp, _vp]
_lib.safedit_pcsp_score.argtypes = [_T, _T, _vp, _vp, _i32, _f32, _vp, _vp]
_lib.safedit_mask_is_row_constant.argtypes = [_T, _vp, _vp, _vp]
_lib.safedit_attn_subset.argtypes = [_T, _T, _T, _vp, _i32, _T, _T, _f32, _T, _i32, _vp]
_lib.safedit_attn_subset_ws.argtypes = [_T, _T, _T, _vp, _i32, _T, _T, _f32, _T, _i32, _vp, ctypes.c_size_t, _vp]
_lib.safedit_attn_subset_workspace_size.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                    _i32]
_lib.safedit_attn_subset_workspace_size.restype = ctypes.c_size_t
_lib.safedit_attn_subset_noalloc.argtypes = [_T, _T, _T, _vp, _i32, _T, _T, _f32, _T, _i32, _vp]
_lib.safedit_scatter_state.argtypes = [_T, _T, _i32, _vp, _i32, _vp]
_lib.safedit_gather_rows.argtypes = [_T, _T, _i32, _vp, _i32, _vp]
_lib.safedit_sw_cfg.argtypes = [_T, _T, _vp, _f32, _f32, _T, _vp]
_lib.safedit_stepcache_sw_cfg.argtypes = [_T, _T, _T, _T, _vp, _f32, _f32, _f32, _T, _vp]
_lib.safedit_gemm_bias_act.argtypes = [_T, _T, _vp, _i32, _vp, _T, _vp]
_lib.safedit_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_int32), _vp]
_lib.safedit_status_string.argtypes = [ctypes.c_int]
_lib.safedit_status_string.restype = ctypes.c_char_p
_lib.safedit_kernel_launch_count.restype = ctypes.c_uint64
_lib.safedit_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.safedit_debug_set_wait_limit_ns.restype = ctypes.c_uint64
_lib.safedit_debug_set_index_check.argtypes = [ctypes.c_int32]
_lib.safedit_debug_set_index_check.restype = ctypes.c_int32
for _n in EXPORTED:
    if _n not in ("safedit_status_string", "safedit_kernel_launch_count",
                  "safedit_debug_set_wait_limit_ns", "safedit_debug_set_index_check",
                  "safedit_attn_subset_workspace_size"):
        getattr(_lib, _n).restype = ctypes.c_int


def lib():
    return _lib


def status_string(code: int) -> str:
    return _lib.safedit_status_string(int(code)).decode()


def _check(code, where):
    if code != OK:
        raise SafeditError(code, where)


def tensor_desc(t: torch.Tensor) -> SafeditTensor:
    """Descriptor of a torch tensor (device pointer, dtype, dims, element strides)."""
    if t.dim() < 1 or t.dim() > 4:
        raise ValueError("safedit tensors have 1 to 4 dims")
    d = SafeditTensor()
    d.data = t.data_ptr()
    d.dtype = _DTYPE[t.dtype]
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.dims[i] = t.shape[i]
        d.strides[i] = t.stride(i)
    return d


def _ref(t):
    return None if t is None else ctypes.byref(tensor_desc(t))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ---- entry points (same names as the C ABI) --------------------------------
def safedit_cross_attn_probs(q_img, k_txt, key_valid, batch_index, scale, p_out, stream=None):
    _check(_lib.safedit_cross_attn_probs(_ref(q_img), _ref(k_txt), _ptr(key_valid), int(batch_index),
                                         float(scale), _ref(p_out), _stream(stream)),
           "safedit_cross_attn_probs")


def safedit_partition_accumulate(p, content, score, stream=None):
    _check(_lib.safedit_partition_accumulate(_ref(p), _ptr(content), _ptr(score), _stream(stream)),
           "safedit_partition_accumulate")


def safedit_pcsp_score(q_img, k_txt, key_valid, content, batch_index, scale, score, stream=None):
    _check(_lib.safedit_pcsp_score(_ref(q_img), _ref(k_txt), _ptr(key_valid), _ptr(content),
                                   int(batch_index), float(scale), _ptr(score), _stream(stream)),
           "safedit_pcsp_score")


def safedit_partition_finalize(score, n, k, idx_s, idx_c, s, stream=None):
    _check(_lib.safedit_partition_finalize(_ptr(score), int(n), int(k), _ptr(idx_s), _ptr(idx_c),
                                           _ptr(s), _stream(stream)), "safedit_partition_finalize")


def safedit_mask_is_row_constant(mask, verdict, row_flags=None, stream=None):
    _check(_lib.safedit_mask_is_row_constant(_ref(mask), _ptr(verdict), _ptr(row_flags),
                                             _stream(stream)), "safedit_mask_is_row_constant")


# A NULL row index means "every row" to safedit_attn_subset, while torch hands
# out a null data pointer for an empty tensor: an empty index is passed as this
# non-null address instead (never dereferenced, since n_idx is then 0).
_EMPTY_INDEX = ctypes.c_void_p(16)


def _idx_ptr(idx):
    if idx is not None and idx.numel() == 0:
        return _EMPTY_INDEX
    return _ptr(idx)


def safedit_attn_subset(q, k, v, idx, n_idx, key_pad, bias, scale, out, out_scattered,
                        stream=None):
    _check(_lib.safedit_attn_subset(_ref(q), _ref(k), _ref(v), _idx_ptr(idx), int(n_idx), _ref(key_pad),
                                    _ref(bias), float(scale), _ref(out), int(out_scattered),
                                    _stream(stream)), "safedit_attn_subset")


def safedit_attn_subset_ws(q, k, v, idx, n_idx, key_pad, bias, scale, out, out_scattered, workspace,
                           stream=None):
    """workspace: a device tensor of at least safedit_attn_subset_workspace_size(...)
    bytes, or None when that size is 0."""
    ptr = None if workspace is None else workspace.data_ptr()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.safedit_attn_subset_ws(_ref(q), _ref(k), _ref(v), _idx_ptr(idx), int(n_idx), _ref(key_pad),
                                       _ref(bias), float(scale), _ref(out), int(out_scattered), ptr, nbytes,
                                       _stream(stream)), "safedit_attn_subset_ws")


def safedit_attn_subset_noalloc(q, k, v, idx, n_idx, key_pad, bias, scale, out, out_scattered, stream=None):
    _check(_lib.safedit_attn_subset_noalloc(_ref(q), _ref(k), _ref(v), _idx_ptr(idx), int(n_idx), _ref(key_pad),
                                            _ref(bias), float(scale), _ref(out), int(out_scattered),
                                            _stream(stream)), "safedit_attn_subset_noalloc")


ATTN_NOALLOC_SCRATCH_BYTES = 24 << 20


def safedit_attn_subset_workspace_size(batch, heads, n_rows, n_keys, head_dim) -> int:
    return int(_lib.safedit_attn_subset_workspace_size(int(batch), int(heads), int(n_rows), int(n_keys),
                                                       int(head_dim)))


def _desc_array(ts):
    arr = (SafeditTensor * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = tensor_desc(t)
    return arr


def safedit_scatter_state(src, dst, idx, n_idx, stream=None):
    """src, dst: sequences of tensors (same length, 1..4)."""
    _check(_lib.safedit_scatter_state(_desc_array(src), _desc_array(dst), len(src), _ptr(idx),
                                      int(n_idx), _stream(stream)), "safedit_scatter_state")


def safedit_gather_rows(src, dst, idx, n_idx, stream=None):
    _check(_lib.safedit_gather_rows(_desc_array(src), _desc_array(dst), len(src), _ptr(idx),
                                    int(n_idx), _stream(stream)), "safedit_gather_rows")


def safedit_sw_cfg(eps_c, eps_u, s, gamma_ctx, gamma_sens, out, stream=None):
    _check(_lib.safedit_sw_cfg(_ref(eps_c), _ref(eps_u), _ptr(s), float(gamma_ctx),
                               float(gamma_sens), _ref(out), _stream(stream)), "safedit_sw_cfg")


def safedit_stepcache_sw_cfg(c_a, c_b, u_a, u_b, s, w, gamma_ctx, gamma_sens, out, stream=None):
    _check(_lib.safedit_stepcache_sw_cfg(_ref(c_a), _ref(c_b), _ref(u_a), _ref(u_b), _ptr(s), float(w),
                                         float(gamma_ctx), float(gamma_sens), _ref(out), _stream(stream)),
           "safedit_stepcache_sw_cfg")


def safedit_gemm_bias_act(a, w, bias, act, idx_out, out, stream=None):
    _check(_lib.safedit_gemm_bias_act(_ref(a), _ref(w), _ptr(bias), int(act), _ptr(idx_out), _ref(out),
                                      _stream(stream)),
           "safedit_gemm_bias_act")


def safedit_get_device_status(stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(_lib.safedit_get_device_status(ctypes.byref(v), _stream(stream)),
           "safedit_get_device_status")
    return int(v.value)


def safedit_status_string(code: int) -> str:
    return status_string(code)


def safedit_kernel_launch_count() -> int:
    return int(_lib.safedit_kernel_launch_count())


def safedit_debug_set_wait_limit_ns(ns: int) -> int:
    return int(_lib.safedit_debug_set_wait_limit_ns(int(ns)))


def safedit_debug_set_index_check(on: bool) -> bool:
    return bool(_lib.safedit_debug_set_index_check(1 if on else 0))


def raw_call(name, *args):
    """Direct access to a C entry point with pre-marshalled ctypes arguments
    (used by the host-validation tests, which pass deliberately bad ones)."""
    return getattr(_lib, name)(*args)
