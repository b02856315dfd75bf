"""Fit the odd polynomial used for tanh(y), |y| <= 1/2, on the FMA pipe.

The prefill softmax applies the logit softcap s * tanh(x / s).  When every
|x / s| of a warp's tile is at most 1/2 (the common case: logits far below
the cap) it evaluates tanh(y) ~= y * P(y^2) with P of 4 terms (degree 7,
kTanhC*) or, for caps up to kTanh5MaxCap, 3 terms (degree 5, kTanh5C*),
fitted here for least maximum absolute error on [0, 1/2] (linear
programming on a grid); otherwise it uses the hardware tanh.  Run:
    python masked_grouped_query_b200/csrc/fit_tanh_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(terms=4, n=4001, ymax=0.5):
    y = np.linspace(0.0, ymax, n)
    t = np.tanh(y)
    V = np.stack([y ** (2 * k + 1) for k in range(terms)], axis=1)
    A = np.vstack([np.hstack([V, -np.ones((n, 1))]), np.hstack([-V, -np.ones((n, 1))])])
    b = np.concatenate([t, -t])
    cost = np.zeros(terms + 1)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * terms + [(0, None)])
    c = res.x[:-1]
    err = np.abs(V @ c - t).max()
    return c, err


if __name__ == "__main__":
    for terms in (4, 3):
        c, e = fit(terms=terms)
        print(f"degree {2 * terms - 1}:")
        for k, v in enumerate(c):
            print(f"  c{2 * k + 1} = {np.float32(v).item()!r}f")
        print(f"  max absolute error {e:.3e}")
