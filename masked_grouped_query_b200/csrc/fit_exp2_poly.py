"""Fit the cubic used for 2^f, 0 <= f < 1, on the FMA pipe.

The prefill softmax computes p = 2^y (y <= 8, log2 domain) for every score.
Most go to the hardware ex2; a share of each row runs on the FMA and integer
pipes instead, by the Cody-Waite split y = j + f with j = floor(y) (an add
with round-down of 1.5 * 2^23, which leaves j in the low mantissa bits) and
2^y = 2^j * P(f): P is evaluated by Horner's rule and j is added to the
result's exponent field.  P here is the cubic of least maximum RELATIVE error
on [0, 1] (linear programming on a grid), so the error of p is the same
fraction of p everywhere (about 1e-4, far below the 2^-9 of the bf16 P fed to
the tensor cores).  Run:
    python masked_grouped_query_b200/csrc/fit_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree=3, n=4001):
    f = np.linspace(0.0, 1.0, n)
    t = np.exp2(f)
    V = np.stack([f ** k for k in range(degree + 1)], axis=1)
    # |V c - t| <= e * t  for every grid point; minimise e.
    A = np.vstack([np.hstack([V, -t[:, None]]), np.hstack([-V, -t[:, None]])])
    b = np.concatenate([t, -t])
    cost = np.zeros(degree + 2)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 1) + [(0, None)])
    c = res.x[:-1]
    err = np.abs(V @ c / t - 1.0).max()
    return c, err


if __name__ == "__main__":
    c, e = fit()
    for k, v in enumerate(c):
        print(f"  kExp2C{k} = {np.float32(v).item()!r}f")
    print(f"  max relative error {e:.3e}")
