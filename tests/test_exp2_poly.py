"""The FMA-pipe exp2 of the kernels (exp2_poly in csrc/sm100_ptx.cuh), checked on the CPU.

The coefficients in the header must be the ones csrc/fit_exp2_poly.py fits (a minimax fit of
2^f on [-1/2, 1/2]); a float32 emulation of the kernel's exact sequence of operations must
stay within 1e-4 relative error of 2^x on [-125, 8] (the kernels feed its result, rounded to
bf16 with relative error up to 2^-9, to the tensor cores); below -125, and at -inf (a masked
score), it must return exactly 0, as 2^-inf = 0 does: a masked key carries no weight.
"""

from __future__ import annotations

import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_116_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coeffs():
    with open(os.path.join(CSRC, "sm100_ptx.cuh")) as f:
        text = f.read()
    return [np.float32(float(re.search(rf"kExp2C{k} = ([0-9.e+-]+)f;", text).group(1))) for k in range(4)]


def test_header_coefficients_are_the_fitted_ones():
    fitted = _fit_module().f32_coeffs()
    header = _header_coeffs()
    for a, b in zip(fitted, header):
        assert abs(float(a) - float(b)) <= 2e-7 * abs(float(a)), (a, b)


def test_emulated_error_bound():
    mod = _fit_module()
    c = _header_coeffs()
    xs = np.concatenate([np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float32),
                         np.float32([-0.5, 0.5, -1.5, 1.5, 0.0, -124.5, 7.999])])
    rel = np.abs(mod.exp2_poly_f32(xs, c).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4
    zero = mod.exp2_poly_f32(np.float32([-np.inf, -1000.0, -126.0, -125.001]), c)
    assert (zero == 0).all(), zero
    edge = mod.exp2_poly_f32(np.float32([-125.0]), c)
    assert edge[0] > 0 and abs(float(edge[0]) / 2.0 ** -125 - 1.0) < 1e-4


def test_header_zeroes_below_the_clamp():
    """Both header forms (scalar and pair) select 0 below the clamp from the unclamped input."""
    with open(os.path.join(CSRC, "sm100_ptx.cuh")) as f:
        text = f.read()
    body1 = text[text.index("float exp2_poly(float x_in)"):text.index("// Packed fp32 pair")]
    assert "x_in >= -125.0f ? r : 0.0f" in body1
    body2 = text[text.index("float2 exp2_poly2(float2 x_in)"):text.index("pack_bf16x2")]
    assert "x_in.x >= -125.0f ? rx : 0.0f" in body2 and "x_in.y >= -125.0f ? ry : 0.0f" in body2
