"""Fits the degree-3 polynomial for 2^f on [-0.5, 0.5] used by exp2_poly2 in
common.cuh: the minimax fit of maximum RELATIVE error, solved as a linear
program over 4001 equally spaced points, then checked in float32 Horner form.

    python block_diffusion_attention_fb_b200/csrc/fit_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(deg=3, n=4001):
    f = np.linspace(-0.5, 0.5, n)
    y = 2.0 ** f
    A = np.vstack([f ** i / y for i in range(deg + 1)]).T
    k = deg + 1
    A_ub = np.vstack([np.hstack([A, -np.ones((n, 1))]), np.hstack([-A, -np.ones((n, 1))])])
    b_ub = np.hstack([np.ones(n), -np.ones(n)])
    c = np.zeros(k + 1)
    c[-1] = 1.0
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * k + [(0, None)])
    return res.x[:k].astype(np.float32), float(res.x[-1])


def horner_rel_err(co):
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.full_like(f, co[-1])
    for c in co[-2::-1]:
        p = (p * f + c).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


if __name__ == "__main__":
    co, err = fit()
    print("coefficients c0..c3:", [f"{float(c):.8f}" for c in co])
    print(f"minimax relative error {err:.3e}; float32 Horner {horner_rel_err(co):.3e}")
