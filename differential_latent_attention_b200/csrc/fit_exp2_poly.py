"""Fits the polynomial the prefill softmax uses for part of its exponentials.

exp2(x) is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2];
2^n is applied by adding n to the float's exponent bits and 2^f is a cubic
p(f). The coefficients minimise the maximum relative error of p against 2^f
on a dense grid (discrete Chebyshev approximation solved as a linear program,
min t s.t. |p(f_i) / 2^f_i - 1| <= t), then are rounded to float32. The
result feeds probabilities that are rounded to bf16 (relative step 2^-8), so
a relative error near 1e-4 is far below what the rounding already adds.

Run: python fit_exp2_poly.py  (prints the coefficients and the error bound)
"""
import numpy as np
from scipy.optimize import linprog

DEGREE = 3


def fit(degree=DEGREE, n_points=4001):
    f = np.linspace(-0.5, 0.5, n_points)
    target = np.exp2(f)
    powers = np.vstack([f ** k for k in range(degree + 1)]).T          # [n, d+1]
    scaled = powers / target[:, None]                                  # p(f)/2^f = scaled @ c
    # variables: c_0..c_d, t ; minimise t
    cost = np.zeros(degree + 2)
    cost[-1] = 1.0
    a_ub = np.vstack([np.hstack([scaled, -np.ones((n_points, 1))]),
                      np.hstack([-scaled, -np.ones((n_points, 1))])])
    b_ub = np.concatenate([np.ones(n_points), -np.ones(n_points)])
    res = linprog(cost, A_ub=a_ub, b_ub=b_ub, bounds=[(None, None)] * (degree + 2), method="highs")
    assert res.success, res.message
    return res.x[:-1].astype(np.float32)


def max_rel_error(coeffs, n_points=200001):
    """Max relative error of the float32 Horner evaluation against 2^f in float64."""
    f = np.linspace(-0.5, 0.5, n_points).astype(np.float32)
    p = np.zeros_like(f)
    for c in coeffs[::-1]:
        p = (p * f + np.float32(c)).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for k, v in enumerate(c):
        print(f"c{k} = {float(v)!r}f  ({float(v).hex()})")
    print(f"max relative error (float32 Horner): {max_rel_error(c):.3e}")
