"""Derive the polynomial used by the attention kernels' FMA-pipe exp2.

2^x is evaluated as 2^n * p(f) with n = round(x) and f = x - n in [-1/2, 1/2].
p is the degree-3 polynomial that minimises the maximum RELATIVE error
|p(f) / 2^f - 1| over [-1/2, 1/2] (Chebyshev / minimax approximation), found
by linear programming on a dense grid (minimise e subject to
|p(f_i) - 2^f_i| <= e * 2^f_i). The coefficients are then rounded to float32
and the error of the rounded polynomial, evaluated the way the kernel does it
(float32 Horner with fused multiply-adds), is reported.

Run: python sink_aware_sliding_head_b200/csrc/derive_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def minimax_coeffs(degree=3, n_grid=4001):
    f = np.linspace(-0.5, 0.5, n_grid)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)          # columns f^0 .. f^d
    # variables: c_0..c_d, e ; minimise e
    cost = np.zeros(degree + 2)
    cost[-1] = 1.0
    #  V c - y <= e y   ->   V c - e y <= y
    # -V c + y <= e y   ->  -V c - e y <= -y
    A = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b = np.concatenate([y, -y])
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 1) + [(0, None)],
                  method="highs")
    assert res.success, res.message
    return res.x[:-1], res.x[-1]


if __name__ == "__main__":
    c, e = minimax_coeffs()
    c32 = np.array(c, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.float32(c32[3])
    for ck in (c32[2], c32[1], c32[0]):
        p = (p * f + ck).astype(np.float32)
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    print("minimax relative error (exact coefficients): %.3e" % e)
    print("max relative error (float32 coefficients, float32 Horner): %.3e" % rel.max())
    for k, ck in enumerate(c32):
        print(f"  c{k} = {ck!r:>14}  ({float(ck).hex()})")
