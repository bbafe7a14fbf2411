"""Coefficients of the FMA-pipe exp2 used by the FP8 forward (csrc/fwd_fp8.cuh, exp2_fma).

    python -m exact_io_aware_43_b200.fit_exp2

2^x is evaluated as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody and Waite's
argument reduction: the integer part goes into the exponent field exactly), and 2^f by a cubic
c0 + c1 f + c2 f^2 + c3 f^3 whose coefficients are chosen here to minimise the largest relative
error over [-1/2, 1/2]: a linear programme over a dense grid (minimise e subject to
|p(f_i) / 2^f_i - 1| <= e), solved with scipy, then rounded to float32 and re-evaluated.
Prints the coefficients and the achieved bound, which the GPU test checks the kernel against.
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree=3, n=4001):
    f = np.linspace(-0.5, 0.5, n)
    t = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / t[:, None]   # p(f)/2^f, linear in c
    # variables (c_0..c_degree, e): minimise e with -e <= V c - 1 <= e
    A = np.block([[V, -np.ones((n, 1))], [-V, -np.ones((n, 1))]])
    b = np.concatenate([np.ones(n), -np.ones(n)])
    cost = np.zeros(degree + 2)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 2), method="highs")
    c = res.x[:-1].astype(np.float32)
    ff = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(c[::-1].astype(np.float64), ff)
    return c, float(np.max(np.abs(p / np.exp2(ff) - 1.0)))


if __name__ == "__main__":
    c, err = fit()
    print("coefficients (float32):", ", ".join(f"{x:.10e}" for x in c))
    print("max relative error on [-1/2, 1/2]:", err)
