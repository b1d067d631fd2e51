"""Coefficients of the cubic 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on f in [-1/2, 1/2]
used by the tensor-core kernel's software exp2 (fb_tc_kernel.cuh, exp2_poly).

Method: minimise the maximum relative error |p(f) / 2^f - 1| by iteratively
reweighted least squares on a dense grid (Lawson's algorithm), starting from the
plain least-squares fit.  Run:  python fit_exp2_poly.py
"""
import numpy as np


def fit(deg=3, n=20001, iters=200):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    A = np.vander(f, deg + 1, increasing=True) / y[:, None]  # relative error rows
    b = np.ones_like(f)
    w = np.ones_like(f) / n
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        e = np.abs(A @ c - b)
        w = w * e
        w /= w.sum()
    err = np.max(np.abs(A @ c - b))
    return c, err


if __name__ == "__main__":
    c, err = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v).item()!r}f")
    print("max relative error", err)
