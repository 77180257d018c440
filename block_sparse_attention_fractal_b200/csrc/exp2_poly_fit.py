"""Fits the cubic used by the attention kernel's software exp2.

2^x = 2^n * 2^f with n = rint(x) and f = x - n in [-1/2, 1/2] (Cody-Waite
range reduction); 2^f is approximated by a cubic p(f) whose maximum relative
error over [-1/2, 1/2] is minimised (Lawson's iteratively reweighted least
squares towards the minimax fit, on a dense grid, in float64).  The
coefficients are then rounded to float32, as the kernel uses them.

    python exp2_poly_fit.py      # prints the coefficients and the error
"""
import numpy as np


def fit(degree=3, iters=200, grid=20001):
    f = np.linspace(-0.5, 0.5, grid)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]   # relative error rows
    w = np.full(grid, 1.0 / grid)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    c32 = c.astype(np.float32)
    rel = np.abs(np.polyval(c32[::-1].astype(np.float64), f) / y - 1.0).max()
    return c32, rel


if __name__ == "__main__":
    c, rel = fit()
    for i, ci in enumerate(c):
        print(f"c{i} = {float(ci)!r}f   // {ci.view(np.uint32):#010x}")
    print(f"max relative error on [-1/2, 1/2]: {rel:.3e}")
