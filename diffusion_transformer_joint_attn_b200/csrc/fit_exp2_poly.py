"""Fit the polynomial that stands in for 2^f, f in [-1/2, 1/2], in the
softmax's FMA-pipe exp2 (csrc/softmax_exp2.cuh).

Minimax in RELATIVE error, solved as a linear program on a dense grid:
minimise e subject to |p(f_k) - 2^f_k| <= e * 2^f_k.  The coefficients are
then rounded to fp32 and the relative error of the fp32 Horner evaluation
(fused multiply-adds, as the kernel does it) is measured on 2^20 points.

    python fit_exp2_poly.py [degree]
"""
import sys

import numpy as np
from scipy.optimize import linprog


def fit(degree: int, grid: int = 4001):
    f = np.cos(np.linspace(0, np.pi, grid)) * 0.5          # Chebyshev-spaced points in [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)          # columns f^0 .. f^d
    # variables: c_0..c_d, e ; minimise e
    c = np.zeros(degree + 2)
    c[-1] = 1.0
    A = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b = np.concatenate([y, -y])
    res = linprog(c, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 1) + [(0, None)], method="highs")
    return res.x[:-1], res.x[-1]


def fp32_horner_error(coef):
    c32 = [np.float32(x) for x in coef]
    f = np.linspace(-0.5, 0.5, 1 << 20, dtype=np.float32)
    acc = np.full_like(f, c32[-1])
    for ck in reversed(c32[:-1]):
        acc = (acc.astype(np.float64) * f + np.float64(ck)).astype(np.float32)   # one rounding per fma
    return float(np.max(np.abs(acc / np.exp2(f.astype(np.float64)) - 1)))


if __name__ == "__main__":
    d = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    coef, e = fit(d)
    print("degree", d, "minimax relative error %.3e" % e, "fp32 evaluation %.3e" % fp32_horner_error(coef))
    for k, ck in enumerate(coef):
        print("  c%d = %.9ef  (fp32 %s)" % (k, ck, np.float32(ck).hex() if hasattr(np.float32, 'hex') else float(np.float32(ck))))
