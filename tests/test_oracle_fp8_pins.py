"""Pins for the FP8 part of the oracle (oracle/fp8_e4m3.py), checked against things other than itself.

* the E4M3 decoder against a code table written out by hand from the format's definition
  (tests/golden/e4m3_codes.json) and against torch's float8_e4m3fn conversion of all 256 codes;
* the decoder's order: positive finite codes are strictly increasing, negative codes mirror them;
* the descale factors through invariances of the attention definition: only the product
  scale * q_descale * k_descale enters the scores, v_descale scales O linearly and leaves LSE alone;
* the closed form Q = 0: O is v_descale times the mean of the visible decoded V rows and
  LSE = ln(#visible).
Each planted mistake (a copy of the module with one plausible bug) must fail at least one pin.
"""

from __future__ import annotations

import json
import os
import types

import numpy as np
import pytest
import torch

from oracle import attention_fp64
from oracle import fp8_e4m3 as real_fp8

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _codes(rng, *shape, lo=0x20, hi=0x48):
    """Random finite E4M3 codes with both signs, magnitudes between 0x20 and 0x48 (0.125 .. 4)."""
    mag = rng.integers(lo, hi, size=shape)
    sign = rng.integers(0, 2, size=shape) << 7
    return (mag | sign).astype(np.uint8)


def pin_code_table(impl):
    with open(os.path.join(GOLDEN, "e4m3_codes.json")) as f:
        table = json.load(f)["codes"]
    for code, want in table.items():
        got = float(impl.decode_e4m3(np.uint8(int(code, 16))))
        if want is None:
            assert np.isnan(got), code
        else:
            assert got == want and np.signbit(got) == np.signbit(want), (code, got, want)


def pin_matches_torch_float8(impl):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = impl.decode_e4m3(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])


def pin_order_and_sign(impl):
    pos = impl.decode_e4m3(np.arange(0x00, 0x7F, dtype=np.uint8))
    assert (np.diff(pos) > 0).all() and pos[0] == 0.0 and pos[-1] == impl.E4M3_MAX
    neg = impl.decode_e4m3(np.arange(0x80, 0xFF, dtype=np.uint8))
    assert np.array_equal(neg, -pos)


def pin_descale_invariances(impl):
    rng = np.random.default_rng(31)
    B, N, H, d = 1, 20, 2, 8
    q8, k8, v8 = (_codes(rng, B, N, H, d) for _ in range(3))
    one = np.ones((B, H))
    for causal, wl, wr in [(False, -1, -1), (True, -1, -1), (False, 3, 2)]:
        base_o, base_l = impl.attention_forward_fp8(q8, k8, v8, one, one, one, 0.3, causal, wl, wr)
        o1, l1 = impl.attention_forward_fp8(q8, k8, v8, 2.0 * one, one, one, 0.15, causal, wl, wr)
        o2, l2 = impl.attention_forward_fp8(q8, k8, v8, one, 4.0 * one, one, 0.075, causal, wl, wr)
        o3, l3 = impl.attention_forward_fp8(q8, k8, v8, one, one, 3.0 * one, 0.3, causal, wl, wr)
        for o, lse in ((o1, l1), (o2, l2)):
            assert np.allclose(o, base_o, atol=1e-12, rtol=0) and np.allclose(lse, base_l, atol=1e-12, rtol=0)
        assert np.allclose(o3, 3.0 * base_o, atol=1e-12, rtol=0) and np.allclose(l3, base_l, atol=1e-12, rtol=0)
        # per-head descales act on their own head only
        qd = np.array([[1.0, 2.0]])
        o4, _ = impl.attention_forward_fp8(q8, k8, v8, qd, one, one, 0.3, causal, wl, wr)
        o5, _ = impl.attention_forward_fp8(q8, k8, v8, one, one, one, 0.6, causal, wl, wr)
        assert np.allclose(o4[:, :, 0], base_o[:, :, 0], atol=1e-12, rtol=0)
        assert np.allclose(o4[:, :, 1], o5[:, :, 1], atol=1e-12, rtol=0)


def pin_zero_query_mean_of_values(impl):
    rng = np.random.default_rng(32)
    B, N, H, d = 1, 12, 1, 4
    q8 = np.zeros((B, N, H, d), dtype=np.uint8)
    k8, v8 = _codes(rng, B, N, H, d), _codes(rng, B, N, H, d)
    vd = 0.5
    with open(os.path.join(GOLDEN, "e4m3_codes.json")) as f:
        table = {int(c, 16): x for c, x in json.load(f)["codes"].items()}
    for causal, wl, wr in [(False, -1, -1), (True, -1, -1), (False, 2, 1)]:
        o, lse = impl.attention_forward_fp8(q8, k8, v8, np.ones((1, 1)), np.ones((1, 1)), np.full((1, 1), vd), 0.7,
                                            causal, wl, wr)
        for i in range(N):
            js = [j for j in range(N) if (wl < 0 or j >= i - wl) and (j <= i if causal else (wr < 0 or j <= i + wr))]
            assert abs(lse[0, 0, i] - np.log(len(js))) < 1e-12
            # mean of the visible V rows, decoded through the hand table where it has the code
            vals = np.array([[table.get(int(c), None) for c in v8[0, j, 0]] for j in js], dtype=object)
            ref_rows = np.where(vals == None, real_fp8.decode_e4m3(v8[0, js, 0]), vals).astype(np.float64)  # noqa: E711
            assert np.allclose(o[0, i, 0], vd * ref_rows.mean(axis=0), atol=1e-12, rtol=0)


FP8_PINS = [pin_code_table, pin_matches_torch_float8, pin_order_and_sign, pin_descale_invariances,
            pin_zero_query_mean_of_values]


@pytest.mark.parametrize("pin", FP8_PINS, ids=lambda f: f.__name__)
def test_fp8_oracle_pin(pin):
    pin(real_fp8)


def test_fp8_forward_rows_match_whole_heads():
    rng = np.random.default_rng(33)
    B, N, H, d = 2, 40, 2, 16
    q8, k8, v8 = (_codes(rng, B, N, H, d) for _ in range(3))
    qd, kd, vd = (rng.uniform(0.01, 0.1, (B, H)) for _ in range(3))
    o, lse = real_fp8.attention_forward_fp8(q8, k8, v8, qd, kd, vd, 0.25, True)
    rows = [0, 5, 39]
    o_r, lse_r = real_fp8.forward_rows_fp8(q8, k8, v8, qd, kd, vd, 1, 1, rows, 0.25, True)
    assert np.allclose(o_r, o[1, rows, 1], atol=1e-13, rtol=0) and np.allclose(lse_r, lse[1, 1, rows], atol=1e-13)


MUTANTS = {
    "bias_8": ("E4M3_BIAS = 7", "E4M3_BIAS = 8"),
    "subnormal_exponent": ("subnormal = (man / 8.0) * np.exp2(1 - E4M3_BIAS)",
                           "subnormal = (man / 8.0) * np.exp2(-E4M3_BIAS)"),
    "subnormal_implicit_one": ("val = sign * np.where(exp == 0, subnormal, normal)", "val = sign * normal"),
    "nan_code_finite": ("return np.where((exp == 0xF) & ((c & 0x7) == 0x7), np.nan, val)", "return val"),
    "mantissa_over_16": ("man = (c & 0x7).astype(np.float64)", "man = (c & 0x7).astype(np.float64) / 2.0"),
    "k_descale_dropped": ("k = dequantize(k8, k_descale)", "k = dequantize(k8, np.ones_like(k_descale))"),
    "v_descale_on_scores": ("q = dequantize(q8, q_descale)", "q = dequantize(q8, q_descale * v_descale)"),
    "descale_heads_transposed": ("return vals * ds[:, None, :, None]", "return vals * ds.T[None, :, :, None].swapaxes(0, 2)"),
}


def _mutant(name):
    src_path = real_fp8.__file__
    with open(src_path) as f:
        src = f.read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found"
    mod = types.ModuleType(f"fp8_mutant_{name}")
    mod.__file__ = src_path
    mod.__dict__["attention_fp64"] = attention_fp64
    exec(compile(src.replace(old, new, 1), src_path, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_fp8_planted_mistakes_are_caught(name):
    mod = _mutant(name)
    failed = []
    for pin in FP8_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
