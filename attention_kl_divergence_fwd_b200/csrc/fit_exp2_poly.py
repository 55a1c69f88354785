"""Fit the polynomial behind the kernels' FMA-pipe exp2 (run: python fit_exp2_poly.py).

2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2]  (Cody-Waite style range
reduction; n is taken with the 1.5*2^23 round-to-nearest shifter). 2^f is replaced by the
polynomial p(f) of degree D that minimises max |p(f)/2^f - 1| on [-1/2, 1/2], solved as
a linear program on a dense grid, then rounded to fp32. The script prints the fp32
coefficients and the relative error of the fp32 Horner evaluation (with fused
multiply-adds, as on the GPU) over every fp32 f in [-1/2, 1/2].
"""
import sys

import numpy as np
from scipy.optimize import linprog


def fit(deg, grid=20001):
    f = np.linspace(-0.5, 0.5, grid)
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True)          # columns f^0 .. f^deg
    # variables: c_0..c_deg, t ; minimise t s.t. |V c / y - 1| <= t
    A = V / y[:, None]
    ones = np.ones((grid, 1))
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([np.ones(grid), -np.ones(grid)])
    c = np.zeros(deg + 2)
    c[-1] = 1.0
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (deg + 2), method="highs")
    return res.x[:-1].astype(np.float32), res.x[-1]


def horner_f32(coef, f):
    """fp32 Horner with fused multiply-add (fp64 product + one fp32 rounding per step)."""
    acc = np.full_like(f, coef[-1], dtype=np.float32)
    for c in coef[-2::-1]:
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(c)).astype(np.float32)
    return acc


if __name__ == "__main__":
    for deg in [int(a) for a in sys.argv[1:]] or [3, 5]:
        coef, t = fit(deg)
        bits = np.arange(np.float32(-0.5).view(np.int32) & 0x7FFFFFFF, dtype=np.int64)
        pos = bits[::997].astype(np.int32).view(np.float32)
        f = np.concatenate([-pos, pos, np.float32([0.5, -0.5])]).astype(np.float32)
        rel = np.abs(horner_f32(coef, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)
        print(f"degree {deg}: LP bound {t:.3e}, fp32 Horner max rel err {rel.max():.3e}")
        print("  coefficients (c0..c%d):" % deg, ", ".join(f"{c!r}f" for c in coef.tolist()))
