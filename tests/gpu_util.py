"""Shared helpers of the GPU parity tests (tolerances, comparisons, marshalling).

Tolerances:
  * attention (SRSU rows / dense anchor): relative Frobenius error <= 5e-3 and
    max |error| <= 2e-2 on N(0,1) inputs, over all compared rows;
  * cross-attention probabilities: max |error| <= 1e-5 (fp32 output);
  * SW-CFG: |out - ref| <= 1e-5 * (|u| + |gamma_i| |c - u|) per element
    (relative to the magnitude of the terms, so that cancellation to ~0 is
    not counted as a relative error);
  * partition indices, scatter / gather: bit-exact.
"""
import numpy as np
import torch

ATTN_REL_FRO = 5e-3
ATTN_MAX_ABS = 2e-2
XATTN_MAX_ABS = 1e-5
CFG_REL = 1e-5


def sd():
    from spatially_adaptive_dit_b200 import safedit
    return safedit


def expect_status(code=0):
    torch.cuda.synchronize()
    got = sd().safedit_get_device_status()
    assert got == code, f"device status {got} ({sd().status_string(got)}), expected {code}"


def rel_fro(a, ref):
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-300))


def check_attn(out, ref, what=""):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rf = rel_fro(out, ref)
    mx = float(np.abs(out - ref).max()) if out.size else 0.0
    assert rf <= ATTN_REL_FRO and mx <= ATTN_MAX_ABS, f"{what}: relFro={rf:.3e} maxabs={mx:.3e}"
    return rf, mx


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()
