"""Fits the cubic of the attention kernel's FMA-pipe exp2 (softmax_math.cuh).

    python exp2_poly_fit.py

2^x is evaluated as 2^n * p(f) with n = round(x) and f = x - n in
[-1/2, 1/2] (Cody and Waite's argument reduction).  p is the cubic of
minimax relative error for 2^f on that interval, found with Lawson's
iteratively reweighted least squares: a weighted least-squares fit on a
dense grid whose weights grow where the error is largest, which converges
to the minimax (equioscillating) solution.  The coefficients are rounded to
float32 and the relative error of the float32 cubic is reported.
"""
import numpy as np


def fit(degree: int = 3, points: int = 20001, iters: int = 400):
    f = np.linspace(-0.5, 0.5, points)
    target = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / target[:, None]   # relative error: (p - t) / t
    b = np.ones_like(f)
    w = np.full(points, 1.0 / points)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    c32 = c.astype(np.float32)
    p = np.zeros_like(f, dtype=np.float32)
    for k in range(degree, -1, -1):
        p = p * f.astype(np.float32) + c32[k]
    rel = np.abs(p.astype(np.float64) / target - 1.0).max()
    return c32, rel


if __name__ == "__main__":
    c, rel = fit()
    for k, v in enumerate(c):
        print(f"c{k} = {float(v)!r}f")
    print(f"max relative error of the float32 cubic on [-1/2, 1/2]: {rel:.3e}")
