"""Coefficients of the cubic that the flash-attention softmax uses for part
of its 2^f evaluations (f in [-1/2, 1/2], after rounding the exponent to the
nearest integer).  They minimise the largest relative error of
c0 + c1 f + c2 f^2 + c3 f^3 against 2^f on a dense grid of the interval: a
linear program in (c0, c1, c2, c3, t) minimising t subject to
|p(f_i) / 2^f_i - 1| <= t at every grid point.

Run: python exp2_poly_fit.py   (prints the coefficients as fp32 literals and
the relative error they reach after rounding to fp32)."""

import numpy as np
from scipy.optimize import linprog


def fit(degree: int = 3, points: int = 4001):
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]  # p(f) / 2^f
    n = degree + 1
    # rows: V c - t <= 1 and -V c - t <= -1
    A = np.vstack([np.hstack([V, -np.ones((points, 1))]), np.hstack([-V, -np.ones((points, 1))])])
    b = np.concatenate([np.ones(points), -np.ones(points)])
    cost = np.zeros(n + 1)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * n + [(0, None)], method="highs")
    c = res.x[:n].astype(np.float32)
    fine = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.zeros_like(fine)
    for k in reversed(range(n)):
        p = p * fine + c[k]
    err = np.max(np.abs(p.astype(np.float64) / np.exp2(fine.astype(np.float64)) - 1))
    return c, err


if __name__ == "__main__":
    c, err = fit()
    print(", ".join(f"{v!r}f" for v in c.tolist()), f"  max rel err {err:.3g}")
