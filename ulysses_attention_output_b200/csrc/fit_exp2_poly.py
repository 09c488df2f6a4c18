"""Fit the polynomial behind the FMA-pipe exp2 used by the attention softmax (csrc/attn.cu).

Method (our own, from the textbook construction): Cody-Waite style range reduction
x = n + f with n = round-to-nearest(x) and f in [-1/2, 1/2], then 2^x = 2^n * p(f) where
p is the degree-3 polynomial with p(0) = 1 that minimises the maximum relative error
|p(f) / 2^f - 1| over [-1/2, 1/2].  The minimax problem is solved as a linear program on a
dense grid (scipy.optimize.linprog), which is the discrete form of the Chebyshev
equioscillation problem.  The scale 2^n is applied by adding n to the exponent field.

Run ``python fit_exp2_poly.py`` to print the coefficients (as the float32 hex literals the
kernel uses) and the achieved error; ``tests/test_exp2_poly.py`` re-runs the fit and checks
both the literals in attn.cu and the error bound of the float32 evaluation.
"""
from __future__ import annotations

import numpy as np


def fit(degree: int = 3, n_grid: int = 4001):
    from scipy.optimize import linprog
    f = np.linspace(-0.5, 0.5, n_grid)
    target = np.exp2(f)
    # unknowns: c1..c_degree (c0 fixed to 1) and t; minimise t
    # |(1 + sum_k c_k f^k) / 2^f - 1| <= t
    A = np.stack([f ** k / target for k in range(1, degree + 1)], axis=1)
    b0 = 1.0 / target - 1.0  # contribution of c0 = 1, moved to the right-hand side
    ones = np.ones((n_grid, 1))
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([-b0, b0])
    c = np.zeros(degree + 1)
    c[-1] = 1.0
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (degree + 1), method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    coeffs = np.concatenate([[1.0], res.x[:degree]])
    return coeffs, res.x[degree]


def to_f32_hex(x: float) -> str:
    return "0x%08x" % np.array([x], dtype=np.float32).view(np.uint32)[0]


def eval_f32(coeffs32: np.ndarray, x: np.ndarray) -> np.ndarray:
    """float32 evaluation in the kernel's order: clamp, shifter rounding, Horner with fused
    multiply-adds (emulated by one rounding of the exact float64 result), exponent add."""
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    shifter = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + shifter).astype(np.float32)
    n = (t - shifter).astype(np.float32)
    f = (x - n).astype(np.float32)
    c0, c1, c2, c3 = (np.float32(c) for c in coeffs32)
    p = (f.astype(np.float64) * c3 + c2).astype(np.float32)
    p = (p.astype(np.float64) * f + c1).astype(np.float32)
    p = (p.astype(np.float64) * f + c0).astype(np.float32)
    bits = p.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    coeffs, err = fit()
    c32 = coeffs.astype(np.float32)
    print("coefficients:", ", ".join(f"{c:.9g} ({to_f32_hex(c)})" for c in c32))
    print(f"minimax relative error of the real polynomial: {err:.3e}")
    xs = np.linspace(-126.0, 8.0, 2_000_001)
    rel = np.abs(eval_f32(c32, xs).astype(np.float64) / np.exp2(xs) - 1.0)
    print(f"float32 evaluation, max relative error on [-126, 8]: {rel.max():.3e}")
