"""Pins for the ALiBi bias of the oracle (``alibi`` / ``alibi_slopes`` in oracle/attention_fp64.py).

* a hand-worked fixture (tests/golden/alibi_zero_query.json): with Q = 0 the weights are
  2^-|i-j| for slope ln 2, and LSE = ln(row sum);
* reversing the sequence maps window (a, b) to (b, a) and leaves the result mirrored (the
  bias depends on |i - j| only);
* a very large slope leaves only j = i with weight (O_i = V_i);
* central finite differences of L = sum(dO * O) for the biased backward;
* per-(batch, head) slopes act on their own head.
Each planted mistake must fail at least one pin.
"""

from __future__ import annotations

import json
import os
import types

import numpy as np
import pytest

from oracle import attention_fp64 as real_oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MASKS = [(False, -1, -1), (True, -1, -1), (False, 3, 5), (False, 2, 0)]


def pin_zero_query_fixture(impl):
    with open(os.path.join(GOLDEN, "alibi_zero_query.json")) as f:
        g = json.load(f)
    n, m = g["N"], g["slope"]
    rng = np.random.default_rng(71)
    v = rng.standard_normal((n, 3))
    q, k = np.zeros((n, 3)), rng.standard_normal((n, 3))
    for case in g["cases"]:
        o, lse = impl.head_forward(q, k, v, 0.9, case["causal"], case["win_l"], case["win_r"], alibi=m)
        w = np.asarray(case["weights"], dtype=np.float64) / np.asarray(case["denominators"], dtype=np.float64)[:, None]
        assert np.allclose(o, w @ v, atol=1e-12, rtol=0), case
        assert np.allclose(lse, np.log(case["row_sums"]), atol=1e-12, rtol=0), case


def pin_reversal(impl):
    rng = np.random.default_rng(72)
    n, d = 17, 4
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    for wl, wr in [(-1, -1), (3, 6), (0, 4)]:
        o, lse = impl.head_forward(q, k, v, 0.5, False, wl, wr, alibi=0.37)
        o2, lse2 = impl.head_forward(q[::-1], k[::-1], v[::-1], 0.5, False, wr, wl, alibi=0.37)
        assert np.allclose(o, o2[::-1], atol=1e-12, rtol=0) and np.allclose(lse, lse2[::-1], atol=1e-12, rtol=0)


def pin_large_slope(impl):
    rng = np.random.default_rng(73)
    n, d = 9, 4
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    for causal, wl, wr in MASKS:
        o, _ = impl.head_forward(q, k, v, 0.3, causal, wl, wr, alibi=200.0)
        assert np.allclose(o, v, atol=1e-12, rtol=0)


def pin_finite_differences(impl):
    rng = np.random.default_rng(74)
    n, d, scale, m = 7, 3, 0.8, 0.45
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    for causal, wl, wr in MASKS:
        dq, dk, dv, _ = impl.head_backward(q, k, v, do, scale, causal, wl, wr, alibi=m)

        def loss(qq, kk, vv):
            return float((impl.head_forward(qq, kk, vv, scale, causal, wl, wr, alibi=m)[0] * do).sum())

        h = 1e-6
        for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = [q, k, v]
                args_m = [q, k, v]
                args_p[which], args_m[which] = xp, xm
                num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert np.allclose(g, num, atol=1e-6 * max(1.0, np.abs(num).max()), rtol=1e-6), (causal, wl, wr, which)


def pin_per_head_slopes(impl):
    rng = np.random.default_rng(75)
    B, n, H, d = 2, 11, 3, 4
    q, k, v, do = (rng.standard_normal((B, n, H, d)) for _ in range(4))
    slopes = rng.uniform(0.05, 1.0, (B, H))
    o, lse = impl.attention_forward(q, k, v, 0.6, True, alibi_slopes=slopes)
    g = impl.attention_backward(q, k, v, do, 0.6, True, alibi_slopes=slopes)
    for b in range(B):
        for h in range(H):
            o_h, lse_h = impl.head_forward(q[b, :, h], k[b, :, h], v[b, :, h], 0.6, True, alibi=slopes[b, h])
            assert np.allclose(o[b, :, h], o_h, atol=1e-13, rtol=0) and np.allclose(lse[b, h], lse_h, atol=1e-13)
            g_h = impl.head_backward(q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], 0.6, True, alibi=slopes[b, h])
            for a, r in zip(g[:3], g_h[:3]):
                assert np.allclose(a[b, :, h], r, atol=1e-13, rtol=0)
    rows = [0, 4, 10]
    o_r, lse_r = impl.forward_rows(q, k, v, 1, 2, rows, 0.6, True, alibi_slopes=slopes)
    assert np.allclose(o_r, o[1, rows, 2], atol=1e-13) and np.allclose(lse_r, lse[1, 2, rows], atol=1e-13)


ALIBI_PINS = [pin_zero_query_fixture, pin_reversal, pin_large_slope, pin_finite_differences, pin_per_head_slopes]


@pytest.mark.parametrize("pin", ALIBI_PINS, ids=lambda f: f.__name__)
def test_alibi_pin(pin):
    pin(real_oracle)


MUTANTS = {
    "alibi_sign": ("s = s - alibi * np.abs(", "s = s + alibi * np.abs("),
    "alibi_no_abs": ("np.abs(np.asarray(rows, dtype=np.int64)[:, None] - keys[None, :])",
                     "(np.asarray(rows, dtype=np.int64)[:, None] - keys[None, :])"),
    "alibi_scaled": ("s = s - alibi * np.abs(", "s = s - scale * alibi * np.abs("),
    "alibi_backward_dropped": ("win_r, alibi)\n    p, _ = _softmax_rows(s)", "win_r)\n    p, _ = _softmax_rows(s)"),
    "alibi_slope_batch_ignored": ("np.asarray(alibi_slopes, dtype=np.float64)[b, h]",
                                  "np.asarray(alibi_slopes, dtype=np.float64)[0, h]"),
}


def _mutant(name):
    src_path = real_oracle.__file__
    with open(src_path) as f:
        src = f.read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found"
    mod = types.ModuleType(f"alibi_mutant_{name}")
    mod.__file__ = src_path
    exec(compile(src.replace(old, new, 1), src_path, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_alibi_planted_mistakes_are_caught(name):
    mod = _mutant(name)
    failed = []
    for pin in ALIBI_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
