"""Fits the polynomial used by the FMA-pipe exp2 of the attention kernel.

2^x is split (Cody-Waite range reduction) as x = n + f with n = floor(x) and
f in [0, 1); 2^f is approximated by a degree-3 polynomial p(f) whose
coefficients minimise the maximum relative error on [0, 1] (a minimax fit,
solved here as a linear program on a dense grid -- the discrete form of the
Remez problem), with p(0) = 1 imposed so that 2^n is exact at integers.
The result is scaled by 2^n by adding n to the exponent field.

    python kv_cache_compression_fkv_b200/csrc/fit_exp2_poly.py

prints the coefficients (as float32 hex and decimal) and the error bound that
the GPU test checks.
"""
import numpy as np
from scipy.optimize import linprog

DEG = 3


def fit(deg=DEG, grid=20001):
    f = np.linspace(0.0, 1.0, grid)
    y = np.exp2(f)
    # unknowns: c1..c_deg, t ; minimise t s.t. |(1 + sum c_k f^k)/y - 1| <= t
    A = np.stack([f ** k / y for k in range(1, deg + 1)], axis=1)
    b0 = 1.0 / y - 1.0
    ones = np.ones((grid, 1))
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([-b0, b0])
    c = np.zeros(deg + 1)
    c[-1] = 1.0
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (deg + 1), method="highs")
    coef = np.concatenate([[1.0], res.x[:deg]])
    return coef, res.x[-1]


def horner32(coef, f):
    c = coef.astype(np.float32)
    r = np.full_like(f, c[-1], dtype=np.float32)
    for k in range(len(c) - 2, -1, -1):
        r = (r * f + c[k]).astype(np.float32)
    return r


if __name__ == "__main__":
    coef, t = fit()
    f = np.linspace(0, 1, 1_000_001, dtype=np.float32)
    err = np.max(np.abs(horner32(coef, f) / np.exp2(f.astype(np.float64)) - 1.0))
    for k, c in enumerate(coef.astype(np.float32)):
        print(f"c{k} = {float(c):.9e}  (0x{c.view(np.uint32):08x})")
    print(f"minimax relative error {t:.3e}; in float32 Horner {err:.3e}")
