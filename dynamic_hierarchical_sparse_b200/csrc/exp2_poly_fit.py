"""Fits the degree-3 polynomial behind the FMA-pipe exp2 of the attention kernel.

2^x is split Cody-Waite style into 2^j * 2^f with j = round(x) and
f = x - j in [-1/2, 1/2]; 2^f is approximated by p(f) = c0 + c1 f + c2 f^2 + c3 f^3
whose maximum relative error on [-1/2, 1/2] is minimised with Lawson's
iteratively re-weighted least squares (the minimax limit of weighted L2 fits).

    python exp2_poly_fit.py        # prints the coefficients and the error bound

The printed constants are the ones in exp2_poly.cuh.
"""

import numpy as np


def fit(degree: int = 3, iters: int = 400, grid: int = 20001):
    f = np.linspace(-0.5, 0.5, grid)
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / target[:, None]  # relative error system
    w = np.full(grid, 1.0 / grid)
    coef = None
    for _ in range(iters):
        sw = np.sqrt(w)
        coef, *_ = np.linalg.lstsq(V * sw[:, None], np.ones(grid) * sw, rcond=None)
        err = np.abs(V @ coef - 1.0)
        w = w * err
        w /= w.sum()
    err = np.abs(np.polyval(coef[::-1], f) / target - 1.0)
    return coef, float(err.max())


def emulate_f32(x, coef):
    """The kernel's steps in float32 (round via 1.5*2^23, Horner, exponent add)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    fr = (x - j).astype(np.float32)
    c = [np.float32(v) for v in coef]
    p = c[3]
    for k in (2, 1, 0):
        p = (p * fr + c[k]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


if __name__ == "__main__":
    coef, err = fit()
    print("coefficients c0..c3:", ", ".join("%.9e" % c for c in coef))
    print("max relative error on [-1/2, 1/2]: %.3e" % err)
    xs = np.linspace(-30, 8, 200001).astype(np.float32)
    rel = np.abs(emulate_f32(xs, coef).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1)
    print("float32 emulation, x in [-30, 8]: max relative error %.3e" % rel.max())
