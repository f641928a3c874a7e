"""ctypes front end of the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the benchmark's
CPU-baseline leg import this module; the CUDA library and its Python binding
never do, and this module never imports them.

Inputs may be numpy arrays or torch tensors of any float dtype; they are
widened exactly to float64 (bf16/fp16/fp32 -> double is exact) before the C
code sees them.  All results are float64 numpy arrays (s is float32, indices
int32), following the definitions cited in oracle.c.
"""
import ctypes
import math

import numpy as np

from . import build_oracle

_lib = None
_dp = ctypes.POINTER(ctypes.c_double)
_fp = ctypes.POINTER(ctypes.c_float)
_ip = ctypes.POINTER(ctypes.c_int32)
_up = ctypes.POINTER(ctypes.c_uint8)
_i64 = ctypes.c_int64

ERRORS = {-1: "invalid argument", -2: "index out of range or duplicated",
          -3: "row with no admissible key", -4: "NaN score"}


class OracleError(RuntimeError):
    pass


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_cross_attn_probs.argtypes = [_i64, _i64, _i64, _i64, _dp, _dp, _up, ctypes.c_double, _dp]
        L.oracle_partition_accumulate.argtypes = [_i64, _i64, _i64, _dp, _up, _dp]
        L.oracle_partition_select.argtypes = [_i64, _i64, _dp, _ip, _ip, _fp]
        L.oracle_mask_row_constant.argtypes = [_i64, _i64, _dp, _up]
        L.oracle_mask_row_constant_bool.argtypes = [_i64, _i64, _up, _up]
        L.oracle_attn_subset.argtypes = [_i64, _i64, _i64, _dp, _dp, _dp, _ip, _i64, _dp, _dp,
                                         ctypes.c_double, _dp]
        L.oracle_attn_dense.argtypes = [_i64, _i64, _i64, _dp, _dp, _dp, _dp, _dp, ctypes.c_double, _dp]
        L.oracle_scatter_rows.argtypes = [_i64, _i64, _i64, _up, _up, _ip]
        L.oracle_gather_rows.argtypes = [_i64, _i64, _i64, _up, _up, _ip]
        L.oracle_sw_cfg.argtypes = [_i64, _i64, _dp, _dp, _dp, ctypes.c_double, ctypes.c_double, _dp]
        L.oracle_sw_cfg.restype = None
        L.oracle_stepcache_sw_cfg.argtypes = [_i64, _i64, _dp, _dp, _dp, _dp, _dp, ctypes.c_double,
                                              ctypes.c_double, ctypes.c_double, _dp]
        L.oracle_stepcache_sw_cfg.restype = None
        L.oracle_ffn_cached.argtypes = [_i64, _i64, _i64, _dp, _ip, _i64, _dp, _dp, _dp, _dp, ctypes.c_int, _dp]
        L.oracle_linear_act.argtypes = [_i64, _i64, _i64, _dp, _dp, _dp, ctypes.c_int, _dp]
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def _f64(x):
    """Exact widening of a numpy array / torch tensor to C-contiguous float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        import torch
        x = x.detach().to("cpu", torch.float64).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _u8(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu", torch.uint8).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x).astype(np.uint8))


def _i32(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _check(rc):
    if rc < 0:
        raise OracleError(ERRORS.get(rc, f"oracle error {rc}"))
    return rc


def default_scale(d: int) -> float:
    # Reading: the pages evaluate on PyTorch SDPA, whose default is 1/sqrt(d).
    return 1.0 / math.sqrt(d)


# ---- C1 -------------------------------------------------------------------
def cross_attn_probs(q, k, key_valid, scale=None):
    """q [H,N,d], k [H,L,d], key_valid [L] -> P [H,N,L] (float64)."""
    q, k, kv = _f64(q), _f64(k), _u8(key_valid)
    H, N, d = q.shape
    L = k.shape[1]
    scale = default_scale(d) if not scale else scale
    P = np.empty((H, N, L), dtype=np.float64)
    _check(lib().oracle_cross_attn_probs(H, N, L, d, _p(q, _dp), _p(k, _dp), _p(kv, _up), scale, _p(P, _dp)))
    return P


# ---- C2 -------------------------------------------------------------------
def partition_accumulate(P, content, score=None):
    """score [N] += sum_h sum_{content j} P[h,i,j]; returns the new score."""
    P, c = _f64(P), _u8(content)
    H, N, L = P.shape
    sc = np.zeros(N, dtype=np.float64) if score is None else np.array(_f64(score), copy=True)
    _check(lib().oracle_partition_accumulate(H, N, L, _p(P, _dp), _p(c, _up), _p(sc, _dp)))
    return sc


# ---- C3 + C4 --------------------------------------------------------------
def partition_select(score, k):
    """-> (idx_s [k] int32 ascending, idx_c [N-k] int32 ascending, s [N] float32)."""
    sc = _f64(score)
    N = sc.shape[0]
    idx_s = np.empty(max(k, 0), dtype=np.int32)
    idx_c = np.empty(max(N - k, 0), dtype=np.int32)
    s = np.empty(N, dtype=np.float32)
    _check(lib().oracle_partition_select(N, k, _p(sc, _dp), _p(idx_s, _ip), _p(idx_c, _ip), _p(s, _fp)))
    return idx_s, idx_c, s


# ---- C5 -------------------------------------------------------------------
def mask_row_constant(mask):
    """mask [..., Nk] (float of any width, or bool) -> (verdict 0/1, row_flags [...] uint8)."""
    is_bool = (hasattr(mask, "dtype") and str(mask.dtype) in ("torch.bool", "bool"))
    if is_bool:
        m = _u8(mask)
    else:
        m = _f64(mask)
    shape = m.shape
    cols = shape[-1]
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    flags = np.empty(rows, dtype=np.uint8)
    if is_bool:
        v = lib().oracle_mask_row_constant_bool(rows, cols, _p(m, _up), _p(flags, _up))
    else:
        v = lib().oracle_mask_row_constant(rows, cols, _p(m, _dp), _p(flags, _up))
    _check(v)
    return int(v), flags.reshape(shape[:-1])


# ---- C6 -------------------------------------------------------------------
def attn_subset(q, k, v, idx=None, pad=None, bias_rows=None, scale=None):
    """One (b,h) slice.  q [Nq,d], k/v [N,d], idx [n] or None, pad [N] or None,
    bias_rows [n,N] (bias rows of the requested queries) or None -> out [n,d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Nq, d = q.shape
    N = k.shape[0]
    idx_a = _i32(idx)
    n = Nq if idx_a is None else idx_a.shape[0]
    pad_a, bias_a = _f64(pad), _f64(bias_rows)
    scale = default_scale(d) if not scale else scale
    out = np.empty((n, d), dtype=np.float64)
    _check(lib().oracle_attn_subset(Nq, N, d, _p(q, _dp), _p(k, _dp), _p(v, _dp), _p(idx_a, _ip), n,
                                    _p(pad_a, _dp), _p(bias_a, _dp), scale, _p(out, _dp)))
    return out


def attn_dense(q, k, v, pad=None, bias=None, scale=None):
    """One (b,h) slice, matrix form.  q [Nq,d], k/v [N,d], bias [Nq,N] -> out [Nq,d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Nq, d = q.shape
    N = k.shape[0]
    pad_a, bias_a = _f64(pad), _f64(bias)
    scale = default_scale(d) if not scale else scale
    out = np.empty((Nq, d), dtype=np.float64)
    _check(lib().oracle_attn_dense(Nq, N, d, _p(q, _dp), _p(k, _dp), _p(v, _dp), _p(pad_a, _dp),
                                   _p(bias_a, _dp), scale, _p(out, _dp)))
    return out


# ---- C7 -------------------------------------------------------------------
def _rows_u8(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint8).reshape(a.shape[0], -1)


def scatter_rows(src, dst, idx):
    """Returns a copy of dst [N,...] with dst[idx[r]] = src[r]."""
    src = np.ascontiguousarray(src)
    out = np.array(dst, copy=True, order="C")
    idx_a = _i32(idx)
    s8, d8 = _rows_u8(src), _rows_u8(out)
    if s8.shape[1] != d8.shape[1]:
        raise OracleError("row size mismatch")
    _check(lib().oracle_scatter_rows(idx_a.shape[0], d8.shape[0], d8.shape[1],
                                     _p(s8, _up), _p(d8, _up), _p(idx_a, _ip)))
    return out


def gather_rows(src, idx):
    """Returns dst [n,...] with dst[r] = src[idx[r]]."""
    src = np.ascontiguousarray(src)
    idx_a = _i32(idx)
    out = np.empty((idx_a.shape[0],) + src.shape[1:], dtype=src.dtype)
    s8, d8 = _rows_u8(src), _rows_u8(out)
    _check(lib().oracle_gather_rows(idx_a.shape[0], s8.shape[0], s8.shape[1],
                                    _p(s8, _up), _p(d8, _up), _p(idx_a, _ip)))
    return out


# ---- C8 -------------------------------------------------------------------
def sw_cfg(eps_c, eps_u, s, gamma_ctx, gamma_sens):
    """eps_c, eps_u [N,F]; s [N] -> out [N,F] float64."""
    c, u, s = _f64(eps_c), _f64(eps_u), _f64(s)
    N, F = c.shape
    out = np.empty((N, F), dtype=np.float64)
    lib().oracle_sw_cfg(N, F, _p(c, _dp), _p(u, _dp), _p(s, _dp), float(gamma_ctx), float(gamma_sens),
                        _p(out, _dp))
    return out


# ---- C10 ------------------------------------------------------------------
def stepcache_sw_cfg(c_a, c_b, u_a, u_b, s, w, gamma_ctx, gamma_sens):
    """Extrapolated branches eps_b + w (eps_b - eps_a), then the weighted combine."""
    arrs = [_f64(x) for x in (c_a, c_b, u_a, u_b)]
    sv = _f64(s)
    N, F = arrs[0].shape
    out = np.empty((N, F), dtype=np.float64)
    lib().oracle_stepcache_sw_cfg(N, F, *[_p(a, _dp) for a in arrs], _p(sv, _dp), float(w),
                                  float(gamma_ctx), float(gamma_sens), _p(out, _dp))
    return out


# ---- C11 ------------------------------------------------------------------
def ffn_cached(x, idx, w1, b1, w2, b2, y_cache, act=1):
    """Returns a copy of y_cache [N,D] with rows idx recomputed as
    W2 gelu(W1 x + b1) + b2 (act=0: no activation).  Weights [out, in]."""
    x, w1, w2 = _f64(x), _f64(w1), _f64(w2)
    b1a, b2a = _f64(b1), _f64(b2)
    y = np.array(_f64(y_cache), copy=True)
    N, D = x.shape
    F = w1.shape[0]
    idx_a = _i32(idx)
    n = N if idx_a is None else idx_a.shape[0]
    _check(lib().oracle_ffn_cached(N, D, F, _p(x, _dp), _p(idx_a, _ip), n, _p(w1, _dp), _p(b1a, _dp),
                                   _p(w2, _dp), _p(b2a, _dp), int(act), _p(y, _dp)))
    return y


# ---- C12 ------------------------------------------------------------------
def linear_act(a, w, b=None, act=0):
    """out [M,N] = act(a [M,K] w[N,K]^T + b[N]) in fp64 (act 1 = gelu-tanh)."""
    a, w = _f64(a), _f64(w)
    ba = None if b is None else _f64(b)
    M, K = a.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise OracleError("shape mismatch")
    out = np.empty((M, N), dtype=np.float64)
    _check(lib().oracle_linear_act(M, K, N, _p(a, _dp), _p(w, _dp), _p(ba, _dp), int(act), _p(out, _dp)))
    return out


# ---- C9 -------------------------------------------------------------------
def is_anchor_step(t: int, warmup: int, period: int) -> bool:
    """Schedule reading: warm-up steps are dense; afterwards step t is a dense
    anchor (CAR) when t % period == 0, otherwise an SRSU step."""
    return t < warmup or (t % period == 0)


def trajectory(steps, warmup, period, k, gamma_ctx, gamma_sens):
    """The SRSU / CAR schedule [SAFE-DiT summary, 방법론 2-4], composed from
    C1-C8.  `steps` is a list of per-step dicts of inputs (numpy / torch):
      q, k_full, v_full: [B,H,N,d]; k_s, v_s: [B,H,k,d] (fresh sensitive rows);
      q_img, k_txt: [B,H,N,d] / [B,H,L,d], key_valid [B,L], content [L]
      (warm-up steps); eps_c, eps_u: [N,F].
    Warm-up steps (t < warmup) are dense and accumulate the PCSP score from
    the cond branch (b = 0); the split follows the last warm-up step; then
    step t is an anchor when t % period == 0 (full refresh of K/V/O state),
    otherwise SRSU: K_state[S] <- K_S, V_state[S] <- V_S, O_state[S] <-
    attention of the S rows over the merged state.  Every step ends with the
    guidance combine (global gamma_ctx until the split exists).
    Returns dict(idx_s, s, score, k_state, v_state, o_state, cfg=[per step])."""
    score = None
    idx_s = s = None
    k_state = v_state = o_state = None
    cfg = []
    for t, st in enumerate(steps):
        if t < warmup:
            kv = _u8(st["key_valid"])
            P = cross_attn_probs(_f64(st["q_img"])[0], _f64(st["k_txt"])[0], kv[0])
            score = partition_accumulate(P, st["content"], score)
        if t == warmup - 1:
            idx_s, _, s = partition_select(score, k)
        q = _f64(st["q"])
        B, H, N, d = q.shape
        if is_anchor_step(t, warmup, period):
            k_state = _f64(st["k_full"]).copy()
            v_state = _f64(st["v_full"]).copy()
            o_state = np.empty_like(q)
            for b in range(B):
                for h in range(H):
                    o_state[b, h] = attn_dense(q[b, h], k_state[b, h], v_state[b, h])
        else:
            ks, vs = _f64(st["k_s"]), _f64(st["v_s"])
            for b in range(B):
                for h in range(H):
                    k_state[b, h] = scatter_rows(ks[b, h], k_state[b, h], idx_s)
                    v_state[b, h] = scatter_rows(vs[b, h], v_state[b, h], idx_s)
                    rows = attn_subset(q[b, h], k_state[b, h], v_state[b, h], idx_s)
                    o_state[b, h] = scatter_rows(rows, o_state[b, h], idx_s)
        sv = s if s is not None else np.zeros(N, dtype=np.float32)
        g_sens = gamma_sens if t >= warmup else gamma_ctx
        cfg.append(sw_cfg(st["eps_c"], st["eps_u"], sv, gamma_ctx, g_sens))
    return dict(idx_s=idx_s, s=s, score=score, k_state=k_state, v_state=v_state, o_state=o_state, cfg=cfg)


__all__ = ["OracleError", "lib", "num_threads", "default_scale", "cross_attn_probs",
           "partition_accumulate", "partition_select", "mask_row_constant", "attn_subset",
           "attn_dense", "scatter_rows", "gather_rows", "sw_cfg", "is_anchor_step", "trajectory", "stepcache_sw_cfg", "ffn_cached",
           "linear_act"]
