"""Fits the polynomial used by the software exp2 in sm100.cuh (soft_exp2).

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody and Waite's additive range reduction, here for base 2); 2^f is
approximated by a degree-3 polynomial whose coefficients minimise the maximum
relative error on [-1/2, 1/2].  The fit starts from weighted least squares on
Chebyshev nodes and refines it with Lawson's iteratively reweighted least
squares (a standard route to the minimax fit, see J.-M. Muller, "Elementary
Functions: Algorithms and Implementation", chapter on polynomial
approximation).  Coefficients are then rounded to fp32 and the error of the
rounded polynomial is reported.

    python rank_biased_window_b200/csrc/gen_exp2_poly.py
"""
import numpy as np

DEG = 3


def fit(deg=DEG, iters=200):
    k = np.arange(4000)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / len(k))        # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(iters):                               # Lawson's algorithm (relative error)
        A = V * (w / y)[:, None]
        c, *_ = np.linalg.lstsq(A, w, rcond=None)
        err = np.abs(V @ c - y) / y
        w = w * err
        w /= w.sum()
    return c


def max_rel_err(c32):
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float64)
    p = np.zeros_like(f)
    for ci in reversed(c32.astype(np.float64)):
        p = p * f + ci
    return float(np.max(np.abs(p - np.exp2(f)) / np.exp2(f)))


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci)!r}f")
    print("max relative error on [-1/2, 1/2]:", max_rel_err(c32))
