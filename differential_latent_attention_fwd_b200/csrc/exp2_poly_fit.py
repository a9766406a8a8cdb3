"""Coefficients of the cubic 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2] used by the
prefill attention softmax for the exponentials it evaluates on the FMA pipe.

Method: least squares on a dense grid with weights that are re-scaled by the square root of
the current relative error on every iteration (Lawson's iteration), which converges towards
the minimax (equi-oscillating) relative-error fit.  Run: python exp2_poly_fit.py
"""
import numpy as np


def fit(deg=3, iters=300, n=40001):
    f = np.linspace(-0.5, 0.5, n)
    t = 2.0 ** f
    w = np.ones_like(f)
    V = np.vander(f, deg + 1, increasing=True)
    for _ in range(iters):
        W = w / t
        c, *_ = np.linalg.lstsq(V * W[:, None], t * W, rcond=None)
        err = (V @ c - t) / t
        w = w * np.abs(err) ** 0.5 + 1e-30
        w /= w.sum()
    return c.astype(np.float32)


def max_rel_err_f32(c):
    """Max relative error of the float32 Horner evaluation over [-1/2, 1/2]."""
    f = np.linspace(-0.5, 0.5, 40001)
    x = f.astype(np.float32)
    acc = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        acc = (acc * x + c[k]).astype(np.float32)
    return float(np.abs(acc.astype(np.float64) / 2.0 ** f - 1.0).max())


if __name__ == "__main__":
    c = fit()
    print("coefficients c0..c3:", [repr(float(v)) for v in c])
    print("max relative error (float32 Horner):", max_rel_err_f32(c))
