"""Fit the polynomial that attn_fwd.cuh uses for 2^f on [-1/2, 1/2].

Method: minimax in relative error, solved as a linear program on a dense
grid:
    minimise t  subject to  |p(f_i) - 2^f_i| <= t * 2^f_i  for every grid point,
with p(0) = 1 and p(1/2) = 2 p(-1/2) pinned. Together these make 2^n * p(f)
exact at integers and continuous where the rounding of n switches.

The kernel combines this polynomial with the usual range reduction
x = n + f, n = round(x), and puts 2^n straight into the exponent bits of
the float result (the Cody-Waite style split for exp2). Run this script to
reproduce the coefficients; tests/test_exp2_poly.py checks the error bound
of the values stored in the header.
"""
from __future__ import annotations

import numpy as np
from scipy.optimize import linprog


def fit(degree: int = 3, grid: int = 4001):
    f = np.linspace(-0.5, 0.5, grid)
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)  # columns 1, f, f^2, ...
    n = degree + 1
    # variables: c_0..c_deg, t ; minimise t
    cost = np.zeros(n + 1)
    cost[-1] = 1.0
    A = np.vstack([np.hstack([V, -target[:, None]]), np.hstack([-V, -target[:, None]])])
    b = np.concatenate([target, -target])
    A_eq = np.zeros((2, n + 1))
    A_eq[0, 0] = 1.0                                           # p(0) = 1
    A_eq[1, :n] = 0.5 ** np.arange(n) - 2.0 * (-0.5) ** np.arange(n)  # p(1/2) - 2 p(-1/2) = 0
    b_eq = np.array([1.0, 0.0])
    res = linprog(cost, A_ub=A, b_ub=b, A_eq=A_eq, b_eq=b_eq, bounds=[(None, None)] * (n + 1), method="highs")
    assert res.success, res.message
    return res.x[:n], res.x[-1]


if __name__ == "__main__":
    c, err = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v)!r}  ({v:.17g})")
    print(f"max relative error {err:.3e}")
