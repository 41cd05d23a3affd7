"""Fit the cubic that the prefill kernel uses for part of its 2^x evaluations.

The kernel splits x = n + f with n = round(x) (integer) and f in [-1/2, 1/2],
evaluates 2^f with a cubic p(f) = 1 + f*(c1 + f*(c2 + f*c3)) (Horner, three
fused multiply-adds) and scales by 2^n through the exponent field.  The cubic
is a minimax fit in relative error with p(0) = 1 fixed, found here by a
Remez-style exchange on the three free coefficients (Muller, "Elementary
Functions", ch. 3).  Run:  python fit_exp2_poly.py
"""

import numpy as np


def fit(iters=30):
    # Start from least squares on Chebyshev nodes, then equalise the relative
    # error at the extrema (exchange) by weighted least squares on a fine grid.
    f = np.cos(np.linspace(0, np.pi, 2001)) * 0.5
    target = np.exp2(f)
    w = 1.0 / target
    for _ in range(iters):
        A = np.stack([f, f ** 2, f ** 3], axis=1) * w[:, None]
        b = (target - 1.0) * w
        c, *_ = np.linalg.lstsq(A, b, rcond=None)
        err = (1.0 + f * (c[0] + f * (c[1] + f * c[2]))) / target - 1.0
        w = w * (1.0 + 50.0 * np.abs(err) / np.max(np.abs(err)))
    return c


def max_rel_error(c, n=200001):
    f = np.linspace(-0.5, 0.5, n)
    p = 1.0 + f * (c[0] + f * (c[1] + f * c[2]))
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    print("c1 = %.9ef, c2 = %.9ef, c3 = %.9ef" % tuple(float(x) for x in c32))
    print("max relative error on [-1/2, 1/2]: %.3e" % max_rel_error(c32.astype(np.float64)))
