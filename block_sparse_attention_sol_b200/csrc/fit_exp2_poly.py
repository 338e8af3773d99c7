"""Derives the exp2 polynomial used by the attention kernel's FMA-pipe exponential.

2^x = 2^n * 2^f with n = floor(x), f in [0, 1).  2^f is approximated by
p(f) = 1 + c1 f + c2 f^2 + c3 f^3 whose coefficients minimise the maximum
relative error on [0, 1] (a linear program over a dense grid).  The constant
term is fixed at 1 so that p(0) is exact.  Run:  python fit_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(deg=3, points=4001):
    f = np.linspace(0.0, 1.0, points)
    y = 2.0 ** f
    A = np.stack([f ** k / y for k in range(1, deg + 1)], axis=1)
    b0 = 1.0 / y - 1.0
    ones = np.ones((points, 1))
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([-b0, b0])
    res = linprog(np.r_[np.zeros(deg), 1.0], A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * deg + [(0, None)])
    return res.x[:deg].astype(np.float32), res.x[-1]


if __name__ == "__main__":
    c, t = fit()
    print("max relative error %.3e" % t)
    for i, v in enumerate(c, 1):
        print(f"c{i} = {float(v).hex()}f  // {float(v)!r}")
