"""Coefficients of the polynomial 2^f ~ 1 + c1 f + ... + cn f^n on [0, 1).

The kernels evaluate part of their base-2 exponentials on the FMA pipe
instead of the special-function unit: x = j + f with j = floor(x) (Cody and
Waite's additive range reduction), 2^f from this polynomial, and 2^j added
into the exponent field.  The constant term is pinned to 1 so that 2^j comes
out exact at f = 0 (and x = -127 yields +0.0).

The remaining coefficients minimise the largest relative error
|p(f) / 2^f - 1| over a dense grid of [0, 1] (a Chebyshev / minimax fit posed
as a linear programme), with the coefficients rounded to fp32 afterwards and
the error re-measured in float64.

    python exp2_poly_fit.py        # prints the coefficients used in common.cuh
"""
from __future__ import annotations

import numpy as np
from scipy.optimize import linprog


def fit(degree: int, grid: int = 4001):
    f = np.linspace(0.0, 1.0, grid)
    y = np.exp2(f)
    # variables: c1..cn, t ; minimise t subject to |1 + sum c_k f^k - y| <= t * y
    A = np.stack([f ** k for k in range(1, degree + 1)], axis=1)
    rhs = y - 1.0
    n = degree
    A_ub = np.vstack([np.hstack([A, -y[:, None]]), np.hstack([-A, -y[:, None]])])
    b_ub = np.concatenate([rhs, -rhs])
    c = np.zeros(n + 1)
    c[-1] = 1.0
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (n + 1), method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    coef = res.x[:n].astype(np.float32)
    ff = np.linspace(0.0, 1.0, 200001)
    p = np.ones_like(ff)
    for k, ck in enumerate(coef, start=1):
        p += float(ck) * ff ** k
    err = np.max(np.abs(p / np.exp2(ff) - 1.0))
    return coef, err


if __name__ == "__main__":
    for deg in (3, 4, 5):
        coef, err = fit(deg)
        cs = ", ".join(f"{float(c):.9e}f" for c in coef)
        print(f"degree {deg}: max rel error {err:.3e}; c1..c{deg} = {cs}")
