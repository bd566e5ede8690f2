"""Derives the polynomial p(f) ~= 2^f on [-1/2, 1/2] used by the attention
kernels to evaluate part of their exp2 calls on the FMA pipe instead of the
special-function unit.

Method: the minimax (Chebyshev) approximation in RELATIVE error, found as a
linear program on a dense grid: minimise t subject to |p(f_i) / 2^f_i - 1| <= t.
The coefficients are then rounded to fp32 and the bound re-measured.

    python gen_exp2_poly.py      # prints the coefficients and the error bound
"""
import numpy as np
from scipy.optimize import linprog

DEGREE = 3


def fit(degree=DEGREE, grid=4001):
    f = np.linspace(-0.5, 0.5, grid)
    y = 2.0 ** f
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]   # p(f) / 2^f
    n = degree + 1
    # variables: c_0..c_degree, t ; minimise t
    cost = np.zeros(n + 1)
    cost[-1] = 1.0
    ones = np.ones((grid, 1))
    A = np.vstack([np.hstack([V, -ones]), np.hstack([-V, -ones])])
    b = np.concatenate([np.ones(grid), -np.ones(grid)])
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * n + [(0, None)], method="highs")
    c = res.x[:n].astype(np.float32)
    fine = np.linspace(-0.5, 0.5, 400001)
    rel = np.abs(np.polyval(c[::-1].astype(np.float64), fine) / 2.0 ** fine - 1).max()
    return c, rel


if __name__ == "__main__":
    c, rel = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v):.9e}f  (0x{np.float32(v).view(np.uint32):08x})")
    print(f"max relative error on [-1/2, 1/2]: {rel:.3e}")
