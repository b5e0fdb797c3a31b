"""Fit of the polynomial behind the kernels' FMA-pipe exp2 (run: python fit_exp2_poly.py).

2^x is computed as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2];
2^f is approximated by p(f) = 1 + c1 f + c2 f^2 + c3 f^3 (p(0) = 1 exactly, so
2^x is exact at integer x), with c1..c3 chosen to minimise the maximum
relative error max |p(f) / 2^f - 1| over the interval.  That minimax problem
is linear in (c1, c2, c3, E) once f is sampled on a dense grid, so it is
solved as a linear program (minimise E subject to -E <= p(f_i)/2^f_i - 1 <= E).
The printed float32 coefficients are the ones in sm100_ptx.cuh
(kExp2C1..kExp2C3); the float32 Horner evaluation error is the bound the
tests check.
"""
import numpy as np
from scipy.optimize import linprog


def fit(n_grid: int = 8001):
    f = np.linspace(-0.5, 0.5, n_grid)
    e = np.exp2(f)
    cols = np.stack([f / e, f ** 2 / e, f ** 3 / e], 1)
    one = np.ones((n_grid, 1))
    a_ub = np.vstack([np.hstack([cols, -one]), np.hstack([-cols, -one])])
    b_ub = np.concatenate([1 - 1 / e, -(1 - 1 / e)])
    r = linprog([0, 0, 0, 1], A_ub=a_ub, b_ub=b_ub, bounds=[(None, None)] * 4, method="highs")
    return r.x[:3], r.x[3]


if __name__ == "__main__":
    c123, err = fit()
    c = np.array([1.0, *c123], dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    e32 = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max()
    print("3 rel err (exact coef)", err, "float32 Horner", e32, "coefs", [float(v) for v in c])
