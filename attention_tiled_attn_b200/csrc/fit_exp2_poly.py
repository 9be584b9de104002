"""Fits the polynomial of the software base-2 exponential used by the prefill softmax.

2^x is evaluated as 2^n * p(f) with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody & Waite style argument reduction); the exponent n is added to the bit
pattern of p(f) as an integer.  p is the degree-3 polynomial with p(0) = 1
that minimises the maximum relative error max |p(f) / 2^f - 1| over
[-1/2, 1/2], found here as a linear program on a dense grid (the discrete
minimax problem), then rounded to float32.

    python attention_tiled_attn_b200/csrc/fit_exp2_poly.py

prints the coefficients (c1, c2, c3 of p(f) = 1 + c1 f + c2 f^2 + c3 f^3) and
the maximum relative error of the float32 coefficients.
"""

import numpy as np
from scipy.optimize import linprog


def fit(degree: int = 3, points: int = 20001):
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    # unknowns c1..cd and e;  minimise e  s.t.  |(1 + sum c_k f^k) / y - 1| <= e
    A = np.stack([f ** k / y for k in range(1, degree + 1)], axis=1)
    b0 = 1.0 / y - 1.0
    ones = np.ones((points, 1))
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([-b0, b0])
    c = np.zeros(degree + 1)
    c[-1] = 1.0
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * degree + [(0, None)], method="highs")
    coef = res.x[:degree].astype(np.float32)
    # max relative error of the float32 coefficients, evaluated in float64
    p = 1.0 + sum(float(coef[k - 1]) * f ** k for k in range(1, degree + 1))
    err = np.max(np.abs(p / y - 1.0))
    return coef, err


if __name__ == "__main__":
    coef, err = fit()
    for k, v in enumerate(coef, start=1):
        print(f"c{k} = {float(v)!r}f   # {float(v).hex()}")
    print(f"max relative error = {err:.3e}")
