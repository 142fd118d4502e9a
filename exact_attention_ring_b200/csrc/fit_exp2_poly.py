"""Fits the polynomial that the attention kernels use for part of their exp2
evaluations (see exp2_poly3x2 in sm100_ptx.cuh): p(r) ~ 2^r on [-1/2, 1/2]
with p(0) = 1 exactly, minimising the largest relative error over a dense grid
(a linear programme; the minimax polynomial of the Chebyshev alternation
theorem up to the grid). Prints the coefficients as float32 hex literals and
the relative error of the float32 Horner evaluation.

    python exact_attention_ring_b200/csrc/fit_exp2_poly.py [degree]
"""
import sys

import numpy as np
from scipy.optimize import linprog


def fit(degree: int, n: int = 4001):
    r = np.linspace(-0.5, 0.5, n)
    f = np.exp2(r)
    # unknowns c1..c_degree and the bound e; c0 = 1 so that 2^0 is exact
    V = np.stack([r ** k for k in range(1, degree + 1)], axis=1) / f[:, None]
    base = 1.0 / f - 1.0  # relative error of the constant term alone
    A = np.block([[V, -np.ones((n, 1))], [-V, -np.ones((n, 1))]])
    b = np.concatenate([-base, base])
    cost = np.zeros(degree + 1)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 1), method="highs")
    assert res.success, res.message
    return np.concatenate([[1.0], res.x[:-1]]).astype(np.float32), res.x[-1]


def horner_f32(c, r):
    p = np.full_like(r, c[-1], dtype=np.float32)
    for k in range(len(c) - 2, -1, -1):
        p = (p * r + c[k]).astype(np.float32)  # the kernel fuses each step (one rounding)
    return p


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = fit(deg)
    r = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    rel = np.abs(horner_f32(c, r).astype(np.float64) / np.exp2(r.astype(np.float64)) - 1.0)
    print(f"degree {deg}: fitted max rel error {e:.3e}, float32 Horner {rel.max():.3e}")
    for k, ck in enumerate(c):
        print(f"c{k} = {float(ck).hex()}  ({ck!r})")
