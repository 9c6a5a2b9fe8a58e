"""Pins for the fp64 oracle: it is checked against things other than itself.

Each pin is a function ``pin_*(impl)`` taking an object with the oracle's
``head_forward``, ``head_backward`` and ``head_probs``. The real oracle must pass
every pin; each planted mistake (a copy of the oracle with one plausible bug,
built on the CPU in ``test_planted_mistakes_are_caught``) must fail at least one.

What the pins rest on:
* closed forms: softmax rows sum to 1; Q = 0 gives the mean of the visible V rows
  and LSE = ln(#visible); causal row 0 gives V_0; a single key gives V;
* hand-derived fixtures under tests/golden/ (two-key softmax; window counts);
* symmetries: joint key/value permutation (full attention), sequence reversal
  mapping window (a, b) to window (b, a); window limits equal to full / causal;
* a second, independent implementation (scalar C loops) on small inputs;
* the tiled online-softmax restatement of the pages, in any block order;
* central finite differences of L = sum(dO * O) for the backward;
* gradient identities: sum_j dV_j = sum_i dO_i, sum_j dK_j = 0, D = rowsum(dO * O).
"""

from __future__ import annotations

import json
import os
import types

import numpy as np
import pytest

from oracle import attention_fp64 as real_oracle
from oracle import online_softmax_fp64, scalar_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MASKS = [(False, -1, -1), (True, -1, -1), (False, 3, 5), (True, 4, -1), (False, 0, -1), (False, 7, 0), (True, 0, 0)]


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _fwd(impl, q, k, v, scale, mask, block_rows=None):
    return impl.head_forward(q, k, v, scale, mask[0], mask[1], mask[2], block_rows=block_rows)


def _bwd(impl, q, k, v, do, scale, mask, block_rows=None):
    return impl.head_backward(q, k, v, do, scale, mask[0], mask[1], mask[2], block_rows=block_rows)


# ----------------------------------------------------------------------------- forward pins

def pin_rows_sum_to_one(impl):
    rng = np.random.default_rng(1)
    n, d = 23, 5
    q, k = _rand(rng, n, d), _rand(rng, n, d)
    for causal, wl, wr in MASKS:
        p = impl.head_probs(q, k, 0.7, causal, wl, wr)
        assert np.allclose(p.sum(axis=1), 1.0, atol=1e-13, rtol=0)
        assert (p >= 0).all()


def pin_zero_query_window_counts(impl):
    with open(os.path.join(GOLDEN, "window_counts.json")) as f:
        fx = json.load(f)
    n = fx["N"]
    rng = np.random.default_rng(2)
    v = _rand(rng, n, 3)
    q = np.zeros((n, 4))
    k = _rand(rng, n, 4)
    for case in fx["cases"]:
        cnt = np.array(case["counts"], dtype=np.float64)
        o, lse = _fwd(impl, q, k, v, 1.3, (case["causal"], case["win_l"], case["win_r"]))
        assert np.allclose(lse, np.log(cnt), atol=1e-13, rtol=0), case
        # O_i is the plain mean of the visible V rows: rebuild it from the counts,
        # using that every listed window is the contiguous run ending or starting at i.
        wl, wr = case["win_l"], (0 if case["causal"] else case["win_r"])
        for i in range(n):
            lo = max(0, i - wl) if wl >= 0 else 0
            hi = min(n - 1, i + wr) if wr >= 0 else n - 1
            assert hi - lo + 1 == cnt[i]
            assert np.allclose(o[i], v[lo:hi + 1].mean(axis=0), atol=1e-13, rtol=0)


def pin_causal_row0_and_single_key(impl):
    rng = np.random.default_rng(3)
    q, k, v = _rand(rng, 9, 6), _rand(rng, 9, 6), _rand(rng, 9, 6)
    o, lse = _fwd(impl, q, k, v, 0.4, (True, -1, -1))
    assert np.allclose(o[0], v[0], atol=1e-14, rtol=0)
    assert abs(lse[0] - 0.4 * float(q[0] @ k[0])) < 1e-13
    o1, lse1 = _fwd(impl, q[:1], k[:1], v[:1], 0.4, (False, -1, -1))
    assert np.allclose(o1, v[:1], atol=1e-14, rtol=0)
    assert abs(lse1[0] - 0.4 * float(q[0] @ k[0])) < 1e-13


def pin_two_key_fixture(impl):
    with open(os.path.join(GOLDEN, "two_key_softmax.json")) as f:
        fx = json.load(f)
    q, k, v = (np.array(fx[x], dtype=np.float64) for x in ("q", "k", "v"))
    o, lse = _fwd(impl, q, k, v, fx["scale"], (False, -1, -1))
    assert np.allclose(o, fx["expected_O"], atol=1e-12, rtol=0)
    assert np.allclose(lse, fx["expected_LSE"], atol=1e-12, rtol=0)
    assert np.allclose(impl.head_probs(q, k, fx["scale"], False, -1, -1), fx["expected_P"], atol=1e-12, rtol=0)


def pin_window_limits(impl):
    rng = np.random.default_rng(4)
    n = 17
    q, k, v = _rand(rng, n, 4), _rand(rng, n, 4), _rand(rng, n, 4)
    full = _fwd(impl, q, k, v, 0.5, (False, -1, -1))
    causal = _fwd(impl, q, k, v, 0.5, (True, -1, -1))
    for a, b in zip(_fwd(impl, q, k, v, 0.5, (False, n - 1, n - 1)), full):
        assert np.allclose(a, b, atol=1e-14, rtol=0)
    for a, b in zip(_fwd(impl, q, k, v, 0.5, (False, n + 5, 0)), causal):
        assert np.allclose(a, b, atol=1e-14, rtol=0)
    for a, b in zip(_fwd(impl, q, k, v, 0.5, (True, n - 1, 3)), causal):
        assert np.allclose(a, b, atol=1e-14, rtol=0)


def pin_sequence_reversal(impl):
    """Reversing the sequence maps window (a, b) onto window (b, a)."""
    rng = np.random.default_rng(5)
    n = 19
    q, k, v = _rand(rng, n, 4), _rand(rng, n, 4), _rand(rng, n, 4)
    r = slice(None, None, -1)
    for a, b in [(3, 6), (0, -1), (-1, 2), (5, 0)]:
        o, lse = _fwd(impl, q, k, v, 0.8, (False, a, b))
        orv, lserv = _fwd(impl, q[r], k[r], v[r], 0.8, (False, b, a))
        assert np.allclose(o, orv[r], atol=1e-13, rtol=0)
        assert np.allclose(lse, lserv[r], atol=1e-13, rtol=0)


def pin_key_permutation(impl):
    rng = np.random.default_rng(6)
    n = 21
    q, k, v = _rand(rng, n, 5), _rand(rng, n, 5), _rand(rng, n, 5)
    perm = rng.permutation(n)
    o, lse = _fwd(impl, q, k, v, 0.6, (False, -1, -1))
    op, lsep = _fwd(impl, q, k[perm], v[perm], 0.6, (False, -1, -1))
    assert np.allclose(o, op, atol=1e-13, rtol=0) and np.allclose(lse, lsep, atol=1e-13, rtol=0)
    oq, lseq = _fwd(impl, q[perm], k, v, 0.6, (False, -1, -1))
    assert np.allclose(o[perm], oq, atol=1e-13, rtol=0) and np.allclose(lse[perm], lseq, atol=1e-13, rtol=0)


def pin_online_blocked(impl):
    rng = np.random.default_rng(7)
    n = 45
    q, k, v = _rand(rng, n, 6) * 3, _rand(rng, n, 6) * 3, _rand(rng, n, 6)
    for mask in MASKS:
        o, lse = _fwd(impl, q, k, v, 0.9, mask)
        nblk = -(-n // 8)
        for trial in range(3):
            order = rng.permutation(nblk) if trial else None
            o2, lse2, lse3 = online_softmax_fp64.head_forward_online(q, k, v, 0.9, *mask, block=8, order=order)
            assert np.allclose(o, o2, atol=1e-12, rtol=0), mask
            assert np.allclose(lse, lse2, atol=1e-12, rtol=0), mask
            assert np.allclose(lse, lse3, atol=1e-12, rtol=0), mask


def pin_scalar_c_forward(impl):
    rng = np.random.default_rng(8)
    b_, n, h_, d = 2, 26, 2, 7
    q, k, v = _rand(rng, b_, n, h_, d), _rand(rng, b_, n, h_, d), _rand(rng, b_, n, h_, d)
    for mask in MASKS:
        o_c, lse_c = scalar_ref.forward(q, k, v, 0.35, *mask)
        for b in range(b_):
            for h in range(h_):
                for br in (None, 5):
                    o, lse = _fwd(impl, q[b, :, h], k[b, :, h], v[b, :, h], 0.35, mask, block_rows=br)
                    assert np.allclose(o, o_c[b, :, h], atol=1e-12, rtol=0), mask
                    assert np.allclose(lse, lse_c[b, h], atol=1e-12, rtol=0), mask


# ----------------------------------------------------------------------------- backward pins

def _loss(impl, q, k, v, do, scale, mask):
    return float((_fwd(impl, q, k, v, scale, mask)[0] * do).sum())


def pin_finite_differences(impl):
    rng = np.random.default_rng(9)
    n, d, scale, h = 11, 4, 0.45, 1e-6
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    for mask in [(False, -1, -1), (True, -1, -1), (False, 2, 3)]:
        dq, dk, dv, _ = _bwd(impl, q, k, v, do, scale, mask)
        for x, g in ((q, dq), (k, dk), (v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                old = x[idx]
                x[idx] = old + h
                lp = _loss(impl, q, k, v, do, scale, mask)
                x[idx] = old - h
                lm = _loss(impl, q, k, v, do, scale, mask)
                x[idx] = old
                num[idx] = (lp - lm) / (2 * h)
            err = np.linalg.norm(num - g) / max(np.linalg.norm(g), 1e-30)
            assert err < 1e-6, (mask, err)


def pin_gradient_identities(impl):
    rng = np.random.default_rng(10)
    n, d = 30, 6
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    for mask in MASKS:
        o, _ = _fwd(impl, q, k, v, 0.55, mask)
        dq, dk, dv, dvec = _bwd(impl, q, k, v, do, 0.55, mask)
        assert np.allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12, rtol=0)
        assert np.allclose(dk.sum(axis=0), 0.0, atol=1e-12, rtol=0)
        assert np.allclose(dvec, (do * o).sum(axis=1), atol=1e-12, rtol=0)


def pin_scalar_c_backward(impl):
    rng = np.random.default_rng(11)
    b_, n, h_, d = 1, 24, 2, 5
    q, k, v, do = (_rand(rng, b_, n, h_, d) for _ in range(4))
    for mask in MASKS:
        gc = scalar_ref.backward(q, k, v, do, 0.6, *mask)
        for h in range(h_):
            for br in (None, 7):
                g = _bwd(impl, q[0, :, h], k[0, :, h], v[0, :, h], do[0, :, h], 0.6, mask, block_rows=br)
                for a, b in zip(g[:3], gc):
                    assert np.allclose(a, b[0, :, h], atol=1e-12, rtol=0), mask


FORWARD_PINS = [pin_rows_sum_to_one, pin_zero_query_window_counts, pin_causal_row0_and_single_key,
                pin_two_key_fixture, pin_window_limits, pin_sequence_reversal, pin_key_permutation,
                pin_online_blocked, pin_scalar_c_forward]
BACKWARD_PINS = [pin_finite_differences, pin_gradient_identities, pin_scalar_c_backward]


@pytest.mark.parametrize("pin", FORWARD_PINS + BACKWARD_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(real_oracle)


def test_scalar_c_agrees_on_tiny_config():
    """The two implementations agree on the tiny forward workload (B1 H2 N128 d64) to 1e-12."""
    from exact_attention_116_b200.inputs import CONFIGS, make_inputs
    cfg = CONFIGS["tiny_fwd"]
    q, k, v, _ = (x.double().numpy() for x in make_inputs(cfg))
    o, lse = real_oracle.attention_forward(q, k, v, cfg.scale, cfg.causal, cfg.win_l, cfg.win_r)
    o_c, lse_c = scalar_ref.forward(q, k, v, cfg.scale, cfg.causal, cfg.win_l, cfg.win_r)
    assert np.abs(o - o_c).max() < 1e-12 and np.abs(lse - lse_c).max() < 1e-12


def test_large_logits_stay_finite():
    """Logits of a few hundred (the x8 window workload) give finite O, LSE and gradients."""
    rng = np.random.default_rng(12)
    n, d = 40, 16
    q, k = _rand(rng, n, d) * 8, _rand(rng, n, d) * 8
    v, do = _rand(rng, n, d), _rand(rng, n, d)
    o, lse = real_oracle.head_forward(q, k, v, 0.25, False, 5, 5)
    g = real_oracle.head_backward(q, k, v, do, 0.25, False, 5, 5)
    assert np.isfinite(o).all() and np.isfinite(lse).all() and all(np.isfinite(x).all() for x in g)
    o2, lse2, _ = online_softmax_fp64.head_forward_online(q, k, v, 0.25, False, 5, 5, block=8)
    assert np.allclose(o, o2, atol=1e-12, rtol=0) and np.allclose(lse, lse2, atol=1e-10, rtol=0)


# ----------------------------------------------------------------------------- planted mistakes

MUTANTS = {
    "left_window_off_by_one": ("vis &= j >= i - win_l", "vis &= j > i - win_l"),
    "right_window_off_by_one": ("vis &= j <= i + wr", "vis &= j < i + wr"),
    "causal_ignored": ("return 0 if causal else int(win_r)", "return int(win_r)"),
    "scale_dropped": ("s = scale * (q[rows] @ k[cols].T)", "s = (q[rows] @ k[cols].T)"),
    "q_k_swapped": ("s = scale * (q[rows] @ k[cols].T)", "s = scale * (k[rows] @ q[cols].T)"),
    "lse_missing_max": ("m_safe + np.log(np.where(dead, 1.0, l))", "np.log(np.where(dead, 1.0, l))"),
    "softmax_column_normalised": ("e / np.where(dead, 1.0, l)[:, None]", "e / np.where(dead, 1.0, l)[None, :]"),
    "key_span_short": ("hi = min(n_keys, (r1 - 1) + wr + 1)", "hi = min(n_keys, (r1 - 1) + wr)"),
    "ds_sign": ("ds = p * (dp - d_i[:, None])", "ds = p * (dp + d_i[:, None])"),
    "ds_drops_D": ("ds = p * (dp - d_i[:, None])", "ds = p * dp"),
    "dk_scale_dropped": ("dk[c0:c1] += scale * (ds.T @ q[r0:r1])", "dk[c0:c1] += (ds.T @ q[r0:r1])"),
    "dq_scale_dropped": ("dq[r0:r1] = scale * (ds @ k[c0:c1])", "dq[r0:r1] = (ds @ k[c0:c1])"),
    "dv_untransposed": ("dv[c0:c1] += p.T @ g", "dv[c0:c1] += p @ g[: p.shape[1]] if p.shape[0] >= p.shape[1] else p.T @ g"),
    "dq_uses_dsT": ("dq[r0:r1] = scale * (ds @ k[c0:c1])", "dq[r0:r1] = scale * (ds.T @ k[r0:r1]) if ds.shape[0] == ds.shape[1] else scale * (ds @ k[c0:c1])"),
}


def _mutant(name):
    src_path = real_oracle.__file__
    with open(src_path) as f:
        src = f.read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    mod.__file__ = src_path
    exec(compile(src.replace(old, new, 1), src_path, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    mod = _mutant(name)
    failed = []
    for pin in FORWARD_PINS + BACKWARD_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
