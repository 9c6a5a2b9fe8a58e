"""Fit the coefficients of the FMA-pipe exp2 used by the kernels (``exp2_poly`` in sm100_ptx.cuh).

Method (Cody-Waite range reduction, then a minimax polynomial):
  2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2];
  2^f ~ c0 + f*(c1 + f*(c2 + f*c3)), the coefficients minimising the maximum RELATIVE error
  on [-1/2, 1/2], found as a linear program on a dense grid (minimise t subject to
  |p(f) - 2^f| <= t * 2^f at every grid point).
  2^j is applied by adding j to the exponent field of p(f).

Run ``python fit_exp2_poly.py`` to print the coefficients as float32 literals and the
achieved error bound. Degree 3 gives a relative error near 9e-5, well under the 2^-9
relative rounding of the bf16 probabilities the kernels feed to the tensor cores.
"""

from __future__ import annotations

import numpy as np
from scipy.optimize import linprog


def fit(degree: int = 3, grid: int = 4001):
    f = np.linspace(-0.5, 0.5, grid)
    y = np.exp2(f)
    # variables: c_0..c_degree, t ; minimise t
    powers = np.stack([f ** k for k in range(degree + 1)], axis=1)
    n = degree + 1
    cost = np.zeros(n + 1)
    cost[-1] = 1.0
    # p(f) - y <= t*y  and  y - p(f) <= t*y
    a_ub = np.vstack([np.hstack([powers, -y[:, None]]), np.hstack([-powers, -y[:, None]])])
    b_ub = np.concatenate([y, -y])
    res = linprog(cost, A_ub=a_ub, b_ub=b_ub, bounds=[(None, None)] * n + [(0, None)], method="highs")
    assert res.success, res.message
    return res.x[:n], res.x[-1]


def f32_coeffs(degree: int = 3):
    c, _ = fit(degree)
    return [np.float32(x) for x in c]


def exp2_poly_f32(x, coeffs):
    """float32 emulation of the kernel's sequence of operations (for the error check)."""
    x_in = np.asarray(x, dtype=np.float32)
    x = np.maximum(x_in, np.float32(-125.0))  # keeps 2^j * p(f) a normal float
    magic = np.float32(12582912.0)  # 1.5 * 2^23: adding it rounds to an integer in the low bits
    t = (x + magic).astype(np.float32)
    j_f = (t - magic).astype(np.float32)
    f = (x - j_f).astype(np.float32)
    c0, c1, c2, c3 = coeffs
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    r = bits.astype(np.int32).view(np.float32)
    return np.where(x_in >= np.float32(-125.0), r, np.float32(0.0))  # below -125 (and -inf): exactly 0


if __name__ == "__main__":
    c, err = fit(3)
    c32 = [np.float32(v) for v in c]
    print("max relative error of the fit: %.3e" % err)
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v):.9e}f  // bits 0x{np.float32(v).view(np.uint32):08x}")
    xs = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    rel = np.abs(exp2_poly_f32(xs, c32).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1.0)
    print("float32 evaluation, max relative error on [-125, 8]: %.3e" % rel.max())
