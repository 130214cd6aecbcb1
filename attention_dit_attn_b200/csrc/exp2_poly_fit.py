"""Fits the cubic used by the kernel's FMA-pipe exp2 (exp2_poly2 in attn_common.cuh).

2^x is split as 2^n * 2^f with n = rint(x), f in [-1/2, 1/2]; 2^f is approximated
by c0 + c1 f + c2 f^2 + c3 f^3 with coefficients chosen to minimise the maximum
relative error on [-1/2, 1/2] (iteratively reweighted least squares on a dense grid,
converging to the equioscillating minimax fit).  Prints the float32 coefficients and
the max relative error of a float32 Horner evaluation.
"""
import numpy as np


def fit(deg: int = 3, iters: int = 200):
    f = np.linspace(-0.5, 0.5, 20001)
    y = 2.0 ** f
    A = np.vander(f, deg + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * (sw / y)[:, None], sw, rcond=None)
        rel = A @ c / y - 1
        w = w * (1 + 50 * np.abs(rel) / np.abs(rel).max())
        w /= w.mean()
    return c.astype(np.float32)


def horner32(c, f):
    p = np.full_like(f, c[-1], dtype=np.float32)
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    return p


if __name__ == "__main__":
    c = fit()
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    err = np.abs(horner32(c, f).astype(np.float64) / 2.0 ** f.astype(np.float64) - 1).max()
    print("coefficients:", [float(x) for x in c], "max rel err: %.3e" % err)
