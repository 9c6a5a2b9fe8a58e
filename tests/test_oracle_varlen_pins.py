"""Pins for the packed variable-length oracle (oracle/varlen_fp64.py):

* one sequence filling the batch equals the plain (pinned) oracle on it;
* a sequence's outputs do not depend on the other sequences' contents (isolation);
* permuting the order of the sequences permutes the outputs, rows and LSE columns alike;
* Q = 0 gives LSE = ln(#visible keys counted inside the sequence) (hand-listed counts for
  lengths 3, 0, 5 under causal masking: 1 2 3 | 1 2 3 4 5);
* empty sequences are allowed and contribute nothing.
Each planted mistake must fail at least one pin.
"""

from __future__ import annotations

import types

import numpy as np
import pytest

from oracle import attention_fp64
from oracle import varlen_fp64 as real_varlen

MASKS = [(False, -1, -1), (True, -1, -1), (False, 2, 1)]


def _pack(rng, lens, H=2, d=3):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    total = int(cu[-1])
    return cu, [rng.standard_normal((total, H, d)) for _ in range(4)]


def pin_single_sequence(impl):
    rng = np.random.default_rng(81)
    cu, (q, k, v, do) = _pack(rng, [13])
    for causal, wl, wr in MASKS:
        o, lse = impl.varlen_forward(q, k, v, cu, 0.6, causal, wl, wr)
        o_ref, lse_ref = attention_fp64.attention_forward(q[None], k[None], v[None], 0.6, causal, wl, wr)
        assert np.allclose(o, o_ref[0], atol=1e-13, rtol=0) and np.allclose(lse, lse_ref[0], atol=1e-13, rtol=0)
        g = impl.varlen_backward(q, k, v, do, cu, 0.6, causal, wl, wr)
        g_ref = attention_fp64.attention_backward(q[None], k[None], v[None], do[None], 0.6, causal, wl, wr)
        for a, r in zip(g, g_ref[:3]):
            assert np.allclose(a, r[0], atol=1e-13, rtol=0)


def pin_isolation(impl):
    rng = np.random.default_rng(82)
    cu, (q, k, v, do) = _pack(rng, [5, 7, 4])
    for causal, wl, wr in MASKS:
        o, lse = impl.varlen_forward(q, k, v, cu, 0.5, causal, wl, wr)
        g = impl.varlen_backward(q, k, v, do, cu, 0.5, causal, wl, wr)
        q2, k2, v2, do2 = (x.copy() for x in (q, k, v, do))
        for x in (q2, k2, v2, do2):
            x[cu[0]:cu[1]] += 3.0  # change sequence 0 only
            x[cu[2]:cu[3]] *= -2.0  # and sequence 2
        o2, lse2 = impl.varlen_forward(q2, k2, v2, cu, 0.5, causal, wl, wr)
        g2 = impl.varlen_backward(q2, k2, v2, do2, cu, 0.5, causal, wl, wr)
        sl = slice(int(cu[1]), int(cu[2]))
        assert np.array_equal(o[sl], o2[sl]) and np.array_equal(lse[:, sl], lse2[:, sl])
        for a, b in zip(g, g2):
            assert np.array_equal(a[sl], b[sl])


def pin_permutation(impl):
    rng = np.random.default_rng(83)
    lens = [4, 6, 3]
    cu, (q, k, v, do) = _pack(rng, lens)
    order = [2, 0, 1]
    parts = lambda x: [x[cu[b]:cu[b + 1]] for b in range(3)]  # noqa: E731
    perm = [np.concatenate([parts(x)[b] for b in order]) for x in (q, k, v, do)]
    cu_p = np.concatenate([[0], np.cumsum([lens[b] for b in order])])
    o, lse = impl.varlen_forward(q, k, v, cu, 0.7, True)
    o_p, lse_p = impl.varlen_forward(*perm[:3], cu_p, 0.7, True)
    g = impl.varlen_backward(q, k, v, do, cu, 0.7, True)
    g_p = impl.varlen_backward(*perm, cu_p, 0.7, True)
    for new_b, old_b in enumerate(order):
        a, b = slice(int(cu_p[new_b]), int(cu_p[new_b + 1])), slice(int(cu[old_b]), int(cu[old_b + 1]))
        assert np.allclose(o_p[a], o[b], atol=1e-14, rtol=0) and np.allclose(lse_p[:, a], lse[:, b], atol=1e-14)
        for x, y in zip(g_p, g):
            assert np.allclose(x[a], y[b], atol=1e-14, rtol=0)


def pin_zero_query_counts(impl):
    rng = np.random.default_rng(84)
    cu, (q, k, v, _) = _pack(rng, [3, 0, 5])
    q[:] = 0.0
    o, lse = impl.varlen_forward(q, k, v, cu, 0.9, True)
    counts = [1, 2, 3, 1, 2, 3, 4, 5]  # listed by hand: positions restart at each sequence
    assert np.allclose(lse[0], np.log(counts), atol=1e-13, rtol=0)
    assert np.allclose(o[4], v[3:5].mean(axis=0), atol=1e-13, rtol=0)


VARLEN_PINS = [pin_single_sequence, pin_isolation, pin_permutation, pin_zero_query_counts]


@pytest.mark.parametrize("pin", VARLEN_PINS, ids=lambda f: f.__name__)
def test_varlen_pin(pin):
    pin(real_varlen)


MUTANTS = {
    "slice_off_by_one": ("ob, lb = attention_fp64.attention_forward(q[None, t0:t1], k[None, t0:t1], v[None, t0:t1],",
                         "ob, lb = attention_fp64.attention_forward(q[None, t0:t1], k[None, max(0, t0 - 1):t1 - 1], v[None, max(0, t0 - 1):t1 - 1],"),
    "whole_batch_keys": ("ob, lb = attention_fp64.attention_forward(q[None, t0:t1], k[None, t0:t1], v[None, t0:t1],",
                         "ob, lb = attention_fp64.attention_forward(q[None, t0:t1], k[None, :t1], v[None, :t1],"),
    "lse_layout": ("        lse[:, t0:t1] = lb[0]", "        lse[:, t0:t1] = lb[0][::-1]"),
    "backward_grads_swapped": ("        for out, gb in zip(grads, g[:3]):", "        for out, gb in zip(grads, g[:3][::-1]):"),
}


def _mutant(name):
    src_path = real_varlen.__file__
    with open(src_path) as f:
        src = f.read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found"
    mod = types.ModuleType(f"varlen_mutant_{name}")
    mod.__file__ = src_path
    exec(compile(src.replace(old, new, 1), src_path, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_varlen_planted_mistakes_are_caught(name):
    mod = _mutant(name)
    failed = []
    for pin in VARLEN_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
