"""Fit of the cubic that evaluates 2^f on the FMA pipe in chunk_attn_kernel.

    python fit_exp2_poly.py        # prints the fp32 coefficients c0..c3 and the errors

The attention softmax computes part of its exponentials as 2^x = 2^r * q(f),
with r = round(x) and f = x - r in [-1/2, 1/2] (vkv_attn_kernel.cuh,
exp2_poly2).  q is the degree-3 polynomial that minimises the maximum
RELATIVE error |q(f) / 2^f - 1| on [-1/2, 1/2], found by Lawson's algorithm
(iteratively reweighted least squares converging to the minimax fit; C. L.
Lawson, 1961) on Chebyshev-spaced points.  The coefficients are rounded to
fp32; the error of the fp32 Horner evaluation is reported beside the exact
one.  The tests (tests/test_exp2_poly.py) re-run this fit and compare it with
the constants in the kernel source.
"""
import numpy as np


def fit(deg=3, n=4001, iters=200):
    f = np.cos(np.linspace(0.0, np.pi, n)) * 0.5
    y = np.exp2(f)
    A = np.vander(f, deg + 1, increasing=True) / y[:, None]  # relative error: (A c - 1) = q / 2^f - 1
    b = np.ones_like(f)
    w = np.ones_like(f) / n
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        r = np.abs(A @ c - b)
        w = w * r
        w /= w.sum()
    return c


def errors(c32):
    """Max relative error of the fp32 coefficients: exact arithmetic, and fp32 Horner."""
    ff = np.linspace(-0.5, 0.5, 200001)
    exact = np.abs(np.polyval(np.asarray(c32, np.float64)[::-1], ff) / np.exp2(ff) - 1).max()
    f32 = ff.astype(np.float32)
    p = np.float32(c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * f32 + np.float32(c32[k])).astype(np.float32)
    horner = np.abs(p.astype(np.float64) / np.exp2(f32.astype(np.float64)) - 1).max()
    return float(exact), float(horner)


def coefficients():
    return [float(x) for x in fit(3).astype(np.float32)]


if __name__ == "__main__":
    c = coefficients()
    print("c0..c3 =", ", ".join(f"{x:.9g}" for x in c))
    print("max relative error: exact %.3g, fp32 Horner %.3g" % errors(c))
