"""The FMA-pipe exp2 used for part of the softmax exponentials: its constants
in common.cuh are the ones the Remez derivation produces, and the whole
scheme (magic-number rounding, polynomial, exponent add), evaluated in
float32, stays within 1e-4 relative of the exact 2^x on the range the
softmax feeds it (x <= 8 after the lazy-rescale max subtraction)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "spatially_adaptive_dit_b200", "csrc")


def _fit():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _device_constants():
    text = open(os.path.join(CSRC, "common.cuh")).read()
    vals = {}
    for i in range(4):
        vals[i] = float(re.search(rf"kExp2C{i}\s*=\s*([0-9.eE+-]+)f;", text).group(1))
    return [vals[i] for i in range(4)]


def test_constants_match_derivation():
    fit = _fit()
    c = fit.remez()
    dev = _device_constants()
    for a, b in zip(c, dev):
        assert np.float32(a) == np.float32(b)


def test_scheme_error_bound():
    fit = _fit()
    c = _device_constants()
    assert fit.max_rel_error(c, lo=-125.0, hi=8.0, n=1_000_001) <= 1e-4
    x = np.array([0.0, 1.0, -1.0, 8.0, -0.5, 0.5, -20.25], dtype=np.float32)
    got = fit.scheme_f32(x, c).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1) <= 1e-4)
    # very negative inputs clamp to a tiny non-negative value, never garbage
    tiny = fit.scheme_f32(np.array([-1e30, -500.0, -127.0, -np.inf], dtype=np.float32), c)
    assert np.all((tiny >= 0) & (tiny < 1e-37))
