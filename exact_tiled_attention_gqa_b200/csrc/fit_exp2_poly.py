"""Coefficients of the FMA-pipe exp2 used by the prefill softmax.

2^t = 2^j * 2^f with j = round(t) and f = t - j in [-1/2, 1/2] (Cody-Waite
style range reduction); 2^f is approximated by a cubic p(f) = c0 + c1 f +
c2 f^2 + c3 f^3 chosen to minimise the maximum *relative* error on
[-1/2, 1/2].  The minimax fit is computed with Lawson's algorithm
(iteratively re-weighted least squares, whose weights converge to the
equioscillating minimax solution).  Run this file to print the coefficients
and the error bound that prefill_sm100.cuh quotes.
"""
import numpy as np


def fit(degree=3, n=4001, iters=400):
    f = np.cos(np.linspace(0, np.pi, n)) * 0.5          # Chebyshev-spaced points on [-1/2, 1/2]
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / target[:, None]   # relative-error system
    w = np.full(n, 1.0 / n)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], np.ones(n) * sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c


def max_rel_err_f32(c):
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    cc = c.astype(np.float32)
    p = ((cc[3] * f + cc[2]) * f + cc[1]) * f + cc[0]
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for i, ci in enumerate(c):
        print(f"c{i} = {np.float32(ci)!r}  ({float(np.float32(ci)).hex()})")
    print("max relative error (fp32 Horner):", max_rel_err_f32(c))
