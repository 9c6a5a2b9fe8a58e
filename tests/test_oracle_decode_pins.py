"""Pins for the paged-KV decode oracle (oracle/decode_paged_fp64.py), checked against things
other than itself:

* hand-listed visible-key counts with Q = 0 (tests/golden/decode_window_counts.json): LSE is
  ln(count) and O the mean of the visible V rows, for ragged sequence lengths;
* the pinned training-path oracle: with Sq = seqlen every position is a query row, and the
  result must equal attention_forward on the contiguous sequence; with Sq < seqlen the rows
  must equal the last Sq rows of that result (the new tokens are the newest positions);
* page placement does not matter: shuffling the pages in the cache while updating the block
  table gives the same result, and so does a larger page size.
Each planted mistake (a copy of the module with one plausible bug) must fail at least one pin.
"""

from __future__ import annotations

import json
import os
import types

import numpy as np
import pytest

from oracle import attention_fp64
from oracle import decode_paged_fp64 as real_decode

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MASKS = [(False, -1, -1), (True, -1, -1), (False, 3, 2), (True, 5, -1), (False, 0, 0)]


def paged(rng, seqs, page_size, shuffle=True):
    """Write contiguous (N_b, H, d) sequences into a page pool; returns (cache, block_table)."""
    H, d = seqs[0].shape[1:]
    pages_per = [(len(s) + page_size - 1) // page_size for s in seqs]
    total = sum(pages_per) + 3  # a few pages nobody uses
    order = rng.permutation(total) if shuffle else np.arange(total)
    cache = rng.standard_normal((total, page_size, H, d)) * 100.0  # junk where nothing is written
    table = np.full((len(seqs), max(pages_per) + 2), -1, dtype=np.int32)
    nxt = 0
    for b, s in enumerate(seqs):
        for p in range(pages_per[b]):
            pg = int(order[nxt])
            nxt += 1
            table[b, p] = pg
            rows = s[p * page_size:(p + 1) * page_size]
            cache[pg, :len(rows)] = rows
    return cache, table


def pin_window_counts(impl):
    with open(os.path.join(GOLDEN, "decode_window_counts.json")) as f:
        g = json.load(f)
    rng = np.random.default_rng(51)
    H, d, Sq = 2, 3, g["Sq"]
    vs = [rng.standard_normal((n, H, d)) for n in g["seqlens"]]
    ks = [rng.standard_normal((n, H, d)) for n in g["seqlens"]]
    kc, table = paged(np.random.default_rng(9), ks, 4)
    vc, table_v = paged(np.random.default_rng(9), vs, 4)  # same page order: same generator state
    assert np.array_equal(table, table_v)
    q = np.zeros((len(vs), Sq, H, d))
    for case in g["cases"]:
        o, lse = impl.decode_forward(q, kc, vc, table, g["seqlens"], 0.5, case["causal"], case["win_l"],
                                     case["win_r"])
        for b, n in enumerate(g["seqlens"]):
            for i in range(Sq):
                cnt = case["counts"][b][i]
                pos = n - Sq + i
                assert abs(lse[b, 0, i] - np.log(cnt)) < 1e-12, (case, b, i)
                wr = 0 if case["causal"] else case["win_r"]
                lo = max(0, pos - case["win_l"]) if case["win_l"] >= 0 else 0
                hi = min(n - 1, pos + wr) if wr >= 0 else n - 1
                assert hi - lo + 1 == cnt
                assert np.allclose(o[b, i], vs[b][lo:hi + 1].mean(axis=0), atol=1e-12, rtol=0)


def pin_matches_training_path(impl):
    rng = np.random.default_rng(52)
    H, d = 2, 5
    lens = [13, 7, 20]
    qs = [rng.standard_normal((n, H, d)) for n in lens]
    ks = [rng.standard_normal((n, H, d)) for n in lens]
    vs = [rng.standard_normal((n, H, d)) for n in lens]
    kc, table = paged(np.random.default_rng(1), ks, 4)
    vc, _ = paged(np.random.default_rng(1), vs, 4)
    for causal, wl, wr in MASKS:
        for Sq in (1, 3, 7):
            q = np.stack([x[n - Sq:] for x, n in zip(qs, lens)])
            o, lse = impl.decode_forward(q, kc, vc, table, lens, 0.4, causal, wl, wr)
            for b, n in enumerate(lens):
                o_ref, lse_ref = attention_fp64.attention_forward(qs[b][None], ks[b][None], vs[b][None], 0.4,
                                                                  causal, wl, wr)
                assert np.allclose(o[b], o_ref[0, n - Sq:], atol=1e-12, rtol=0), (causal, wl, wr, Sq, b)
                assert np.allclose(lse[b], lse_ref[0][:, n - Sq:], atol=1e-12, rtol=0)
        # every position a query row
        b, n = 1, lens[1]
        q = qs[b][None]
        o, lse = impl.decode_forward(q, kc[:, :, :, :], vc, table[b:b + 1], [n], 0.4, causal, wl, wr)
        o_ref, lse_ref = attention_fp64.attention_forward(qs[b][None], ks[b][None], vs[b][None], 0.4, causal, wl, wr)
        assert np.allclose(o, o_ref, atol=1e-12, rtol=0) and np.allclose(lse, lse_ref, atol=1e-12, rtol=0)


def pin_page_placement(impl):
    rng = np.random.default_rng(53)
    H, d, Sq = 1, 4, 2
    lens = [9, 16, 5]
    ks = [rng.standard_normal((n, H, d)) for n in lens]
    vs = [rng.standard_normal((n, H, d)) for n in lens]
    q = rng.standard_normal((len(lens), Sq, H, d))
    ref = None
    for seed, page in ((2, 4), (3, 4), (4, 8), (5, 1)):
        kc, table = paged(np.random.default_rng(seed), ks, page, shuffle=seed != 2)
        vc, _ = paged(np.random.default_rng(seed), vs, page, shuffle=seed != 2)
        out = impl.decode_forward(q, kc, vc, table, lens, 0.7, True)
        if ref is None:
            ref = out
        assert np.allclose(out[0], ref[0], atol=1e-12, rtol=0) and np.allclose(out[1], ref[1], atol=1e-12, rtol=0)


def pin_empty_and_short_sequences(impl):
    """A sequence without keys gives O = 0 and LSE = -inf; with fewer keys than Sq the rows
    before its first key see nothing under causal masking."""
    rng = np.random.default_rng(54)
    H, d, Sq = 1, 4, 3
    lens = [0, 2, 5]
    ks = [rng.standard_normal((max(n, 1), H, d))[:n] for n in lens]
    vs = [rng.standard_normal((max(n, 1), H, d))[:n] for n in lens]
    kc, table = paged(np.random.default_rng(6), [k if len(k) else np.zeros((1, H, d)) for k in ks], 4)
    vc, _ = paged(np.random.default_rng(6), [v if len(v) else np.zeros((1, H, d)) for v in vs], 4)
    q = rng.standard_normal((3, Sq, H, d))
    o, lse = impl.decode_forward(q, kc, vc, table, lens, 0.5, True)
    assert (o[0] == 0).all() and np.isneginf(lse[0]).all()
    # sequence 1: positions -1, 0, 1 -> row 0 sees nothing, row 1 sees key 0, row 2 keys 0..1
    assert (o[1, 0] == 0).all() and np.isneginf(lse[1, 0, 0])
    assert np.allclose(o[1, 1], vs[1][0], atol=1e-12, rtol=0)
    assert abs(lse[1, 0, 1] - 0.5 * float(q[1, 1, 0] @ ks[1][0, 0])) < 1e-12


def pin_append_new_rows(impl):
    """Appending the new tokens' rows gives the training-path result of the sequences that end
    with them; appending the rows the cache already holds changes nothing."""
    rng = np.random.default_rng(55)
    H, d, Sq = 2, 4, 3
    lens = [11, 6]
    qs = [rng.standard_normal((n, H, d)) for n in lens]
    ks = [rng.standard_normal((n, H, d)) for n in lens]
    vs = [rng.standard_normal((n, H, d)) for n in lens]
    junk_k = [x.copy() for x in ks]
    junk_v = [x.copy() for x in vs]
    for x in junk_k + junk_v:
        x[-Sq:] = 1e3  # the cache does not yet hold the new rows
    kc, table = paged(np.random.default_rng(8), junk_k, 4)
    vc, _ = paged(np.random.default_rng(8), junk_v, 4)
    q = np.stack([x[-Sq:] for x in qs])
    k_new = np.stack([x[-Sq:] for x in ks])
    v_new = np.stack([x[-Sq:] for x in vs])
    for causal, wl, wr in MASKS:
        o, lse = impl.decode_forward(q, kc, vc, table, lens, 0.3, causal, wl, wr, k_new=k_new, v_new=v_new)
        for b, n in enumerate(lens):
            o_ref, lse_ref = attention_fp64.attention_forward(qs[b][None], ks[b][None], vs[b][None], 0.3, causal, wl, wr)
            assert np.allclose(o[b], o_ref[0, n - Sq:], atol=1e-12, rtol=0), (causal, wl, wr, b)
            assert np.allclose(lse[b], lse_ref[0][:, n - Sq:], atol=1e-12, rtol=0)
    kc2, _ = paged(np.random.default_rng(8), ks, 4)
    vc2, _ = paged(np.random.default_rng(8), vs, 4)
    a = impl.decode_forward(q, kc2, vc2, table, lens, 0.3, True)
    b_ = impl.decode_forward(q, kc2, vc2, table, lens, 0.3, True, k_new=k_new, v_new=v_new)
    assert np.array_equal(a[0], b_[0]) and np.array_equal(a[1], b_[1])


DECODE_PINS = [pin_window_counts, pin_matches_training_path, pin_page_placement, pin_empty_and_short_sequences,
               pin_append_new_rows]


@pytest.mark.parametrize("pin", DECODE_PINS, ids=lambda f: f.__name__)
def test_decode_oracle_pin(pin):
    pin(real_decode)


MUTANTS = {
    "position_off_by_one": ("pos = np.arange(n - Sq, n, dtype=np.int64)", "pos = np.arange(n - Sq + 1, n + 1, dtype=np.int64)"),
    "oldest_rows_as_queries": ("pos = np.arange(n - Sq, n, dtype=np.int64)", "pos = np.arange(0, Sq, dtype=np.int64)"),
    "page_row_swapped": ("cache[int(block_table[b, j // page_size]), j % page_size]",
                         "cache[int(block_table[b, j % page_size]), j // page_size]"),
    "block_table_ignored": ("cache[int(block_table[b, j // page_size]), j % page_size]",
                            "cache[j // page_size, j % page_size]"),
    "seqlen_ignored": ("n = int(seqlens[b])", "n = int(np.max(seqlens))"),
    "append_shifted": ("pos = int(seqlens[b]) - Sq + i\n", "pos = int(seqlens[b]) - Sq + i + 1\n"),
    "append_page_row_swapped": ("out[int(block_table[b, pos // page_size]), pos % page_size] = rows[b, i]",
                                "out[int(block_table[b, pos % page_size]), pos // page_size] = rows[b, i]"),
    "scale_dropped": ("s = np.where(vis, scale * (q[b, :, h] @ k[:, h].T), -np.inf)",
                      "s = np.where(vis, (q[b, :, h] @ k[:, h].T), -np.inf)"),
}


def _mutant(name):
    src_path = real_decode.__file__
    with open(src_path) as f:
        src = f.read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found"
    mod = types.ModuleType(f"decode_mutant_{name}")
    mod.__file__ = src_path
    exec(compile(src.replace(old, new, 1), src_path, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_decode_planted_mistakes_are_caught(name):
    mod = _mutant(name)
    failed = []
    for pin in DECODE_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
