"""Derives the constants of the FMA-pipe exp2 used by attn.cu for part of the
softmax exponentials (the rest go to the MUFU ex2 unit).

Scheme: 2^x = 2^j * 2^f with j = round(x) (via the 1.5 * 2^23 magic add, so
j also sits in the low mantissa bits of t = x + magic), f = x - j in
[-1/2, 1/2], 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3, and the 2^j scaling done by
adding (bits(t) << 23) to the bit pattern of the polynomial value.

The coefficients minimise the maximum *relative* error on [-1/2, 1/2]
(Remez exchange).  Run: python exp2_poly_fit.py  -> prints the constants and
the error of the whole scheme evaluated in float32.
"""
import numpy as np

DEG = 3
MAGIC = 12582912.0  # 1.5 * 2^23


def remez(deg=DEG, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    xs = np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (hi - lo) / 2 + (lo + hi) / 2
    grid = np.linspace(lo, hi, 200001)
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(xs))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        segs = np.split(np.arange(len(grid)), np.nonzero(np.diff(np.sign(err)))[0] + 1)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segs]
        if len(ext) != n:
            break
        xs = grid[ext]
    return c


def scheme_f32(x, c):
    """The device arithmetic, in float32 (fma rounding modelled as two steps)."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    mag = np.float32(MAGIC)
    t = (x + mag).astype(np.float32)
    j = (t - mag).astype(np.float32)
    f = (x - j).astype(np.float32)
    c32 = [np.float32(v) for v in c]
    p = c32[3]
    for k in (2, 1, 0):
        p = (p * f + c32[k]).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def max_rel_error(c, lo=-125.0, hi=8.0, n=2000001):
    x = np.linspace(lo, hi, n).astype(np.float32)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(scheme_f32(x, c) - ref) / ref))


if __name__ == "__main__":
    c = remez()
    for i, v in enumerate(c):
        print(f"c{i} = {float(np.float32(v)):.9g}f")
    print("max relative error of the scheme on [-125, 8]:", max_rel_error(c))
