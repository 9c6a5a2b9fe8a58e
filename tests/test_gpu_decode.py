"""GPU parity of the paged-KV decode (fa_decode_paged, through the C ABI) against the fp64 oracle.

The kernel computes Q K^T and P V with tcgen05 (fp32 accumulation), P rounded to bf16 and O
divided by the sum of the rounded weights, as the training forward does, so the forward's
tolerances apply: per element |ΔO| <= 1e-2 + half a bf16 ulp of O and max |ΔLSE| <= 1e-3. Cases cover
ragged lengths (empty, shorter than Sq, one key, page and tile boundaries), causal / window /
full masks, Sq = 1..8, page sizes 64..512, piece counts 1, automatic and more pieces than tiles,
pieces that span several sequences and sequences spread over several pieces, and the full
decode workloads compared row by row.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_116_b200 as fa
from exact_attention_116_b200.inputs import DECODE_CONFIGS, DecodeConfig, make_decode_inputs
from oracle import decode_paged_fp64 as oracle_dec
from parity import assert_fwd_close

pytestmark = pytest.mark.gpu


def run(q, kc, vc, table, lens, scale, causal, win, splits):
    dev = [t.cuda() for t in (q, kc, vc, table, lens)]
    o, lse = fa.attention_decode_paged(*dev, scale, causal, win, splits)
    fa.check()
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def check(cfg, lens=None, splits=0, causal=None, win=None, what=""):
    q, kc, vc, table, seqlens = make_decode_inputs(cfg)
    if lens is not None:
        seqlens = torch.tensor(lens, dtype=torch.int32)
    causal = cfg.causal if causal is None else causal
    win = (cfg.win_l, cfg.win_r) if win is None else win
    o, lse = run(q, kc, vc, table, seqlens, cfg.scale, causal, win, splits)
    o_ref, lse_ref = oracle_dec.decode_forward(q.double().numpy(), kc.double().numpy(), vc.double().numpy(),
                                               table.numpy(), seqlens.numpy(), cfg.scale, causal, *win)
    dead = ~np.isfinite(lse_ref)
    assert np.array_equal(dead, ~np.isfinite(lse)), f"{what}: rows without keys differ"
    assert (o[dead.transpose(0, 2, 1)] == 0).all() if dead.any() else True
    live = ~dead
    for b in range(cfg.B):
        for h in range(cfg.H):
            rows = np.nonzero(live[b, h])[0]
            if len(rows):
                assert_fwd_close(o[b, rows, h], lse[b, h, rows], o_ref[b, rows, h], lse_ref[b, h, rows],
                                 f"{what} b={b} h={h} len={int(seqlens[b])}")


SMALL = DecodeConfig("small", 5, 3, 2, 128, 1, 700, 128, True, seed=61)


@pytest.mark.parametrize("splits", [1, 0, 3, 40])
def test_decode_ragged_lengths_and_splits(splits):
    # empty, fewer keys than Sq, one key, a full 64-key tile, a full page, past a page boundary
    check(SMALL, lens=[0, 2, 1, 128, 257], splits=splits, what=f"splits={splits}")


@pytest.mark.parametrize("causal,win", [(False, (-1, -1)), (True, (-1, -1)), (False, (100, 5)), (True, (70, -1)),
                                        (False, (0, 0))])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_masks(causal, win, d):
    cfg = DecodeConfig("masks", 3, 8, 3, d, 300, 900, 64, causal, seed=62 + d)
    check(cfg, causal=causal, win=win, splits=0, what=f"d={d} causal={causal} win={win}")


@pytest.mark.parametrize("Sq,page", [(1, 64), (4, 512), (8, 192)])
def test_decode_rows_and_page_sizes(Sq, page):
    cfg = DecodeConfig("pages", 4, Sq, 4, 128, 1, 1500, page, True, seed=63 + Sq)
    check(cfg, splits=0, what=f"Sq={Sq} page={page}")


@pytest.mark.parametrize("splits", [1, 0, 3])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Sq", [1, 2, 3, 4, 5, 6, 7, 8])
def test_decode_tensor_core_rows(Sq, d, splits):
    # the rows of the 8-row build: empty, shorter than Sq, one key, one unit, a unit and a key,
    # several pages
    cfg = DecodeConfig("tc_rows", 6, Sq, 2, d, 1, 700, 64, True, seed=70 + Sq + d)
    check(cfg, lens=[0, max(Sq - 2, 0), 1, 64, 65, 700], splits=splits, what=f"Sq={Sq} d={d} splits={splits}")


@pytest.mark.parametrize("Sq", [4, 8])
def test_decode_tensor_core_large_logits(Sq):
    # q scaled by 24: scores spread over tens of units, so a few keys dominate each row and the
    # bf16 rounding of their weights moves O unless O is divided by the rounded weights
    cfg = DecodeConfig("tc_big", 3, Sq, 2, 128, 1, 500, 128, False, seed=80 + Sq)
    q, kc, vc, table, seqlens = make_decode_inputs(cfg)
    q = (q.float() * 24.0).to(torch.bfloat16)
    o, lse = run(q, kc, vc, table, seqlens, cfg.scale, False, (-1, -1), 0)
    o_ref, lse_ref = oracle_dec.decode_forward(q.double().numpy(), kc.double().numpy(), vc.double().numpy(),
                                               table.numpy(), seqlens.numpy(), cfg.scale, False, -1, -1)
    for b in range(cfg.B):
        for h in range(cfg.H):
            assert_fwd_close(o[b, :, h], lse[b, h], o_ref[b, :, h], lse_ref[b, h], f"large logits b={b} h={h}")


@pytest.mark.parametrize("Sq,d", [(1, 128), (3, 64), (4, 128), (8, 64)])
def test_decode_cache_rows_past_the_end_are_not_used(Sq, d):
    # a cache from an uninitialised allocation: NaN in every row past each sequence's end, in the
    # sequences' own last pages and in the pages no sequence uses
    cfg = DecodeConfig("nan_tail", 4, Sq, 2, d, 1, 600, 128, True, seed=90 + Sq)
    q, kc, vc, table, seqlens = make_decode_inputs(cfg)
    lens = torch.tensor([600, 65, 130, Sq + 7], dtype=torch.int32)
    used = torch.zeros(kc.shape[:2], dtype=torch.bool)
    for b in range(cfg.B):
        for j in range(int(lens[b])):
            used[int(table[b, j // cfg.page_size]), j % cfg.page_size] = True
    kc, vc = kc.clone(), vc.clone()
    kc[~used] = float("nan")
    vc[~used] = float("nan")
    o, lse = run(q, kc, vc, table, lens, cfg.scale, True, (-1, -1), 0)
    o_ref, lse_ref = oracle_dec.decode_forward(q.double().numpy(), kc.double().numpy(), vc.double().numpy(),
                                               table.numpy(), lens.numpy(), cfg.scale, True, -1, -1)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    for b in range(cfg.B):
        for h in range(cfg.H):
            assert_fwd_close(o[b, :, h], lse[b, h], o_ref[b, :, h], lse_ref[b, h], f"b={b} h={h}")


@pytest.mark.parametrize("splits", [1, 2, 7, 0])
def test_decode_pieces_cross_sequences(splits):
    """Pieces of the concatenated tile list that span several short (and empty) sequences, and
    sequences spread over several pieces."""
    lens = [0, 1, 2, 63, 64, 65, 0, 130, 3, 700, 1, 0, 257, 5, 64, 1]
    cfg = DecodeConfig("cross", len(lens), 2, 3, 128, 1, 704, 64, True, seed=69)
    check(cfg, lens=lens, splits=splits, what=f"pieces={splits}")


@pytest.mark.parametrize("splits", [3, 0])
def test_decode_many_sequences(splits):
    """More sequences than threads in a CTA (the tile prefix sums run over several sequences per
    thread), d = 64, a window."""
    g = np.random.default_rng(70)
    lens = [int(x) for x in g.integers(0, 200, size=300)]
    cfg = DecodeConfig("many", 300, 1, 2, 64, 1, 200, 64, False, seed=70)
    check(cfg, lens=lens, splits=splits, causal=False, win=(90, 0), what=f"B=300 pieces={splits}")


def test_decode_split_counts_agree():
    cfg = DecodeConfig("splits", 2, 2, 2, 64, 2000, 3000, 256, True, seed=64)
    q, kc, vc, table, lens = make_decode_inputs(cfg)
    outs = [run(q, kc, vc, table, lens, cfg.scale, True, (-1, -1), s) for s in (1, 2, 5, 0)]
    for o, lse in outs[1:]:
        assert np.abs(o - outs[0][0]).max() < 1e-2 and np.abs(lse - outs[0][1]).max() < 1e-4


@pytest.mark.parametrize("name", ["decode_paged", "decode_paged_sq4"])
def test_decode_workload_all_rows(name):
    cfg = DECODE_CONFIGS[name]
    check(cfg, splits=0, what=name)


def test_decode_out_of_range_length_is_reported_not_read():
    cfg = DecodeConfig("bad", 2, 1, 2, 128, 100, 200, 64, True, seed=65)
    q, kc, vc, table, lens = make_decode_inputs(cfg)
    bad = torch.tensor([int(lens[0]), cfg.max_pages * cfg.page_size + 1], dtype=torch.int32)
    dev = [t.cuda() for t in (q, kc, vc, table, bad)]
    o, lse = fa.attention_decode_paged(*dev, cfg.scale, True, (-1, -1), 1)
    with pytest.raises(fa.FaError) as e:
        fa.check()
    assert e.value.status == 6  # FA_ERR_DEVICE
    assert torch.isinf(lse[1]).all() and (o[1] == 0).all()  # the bad sequence counts as empty
    fa.check()  # the error word was cleared; the context is usable


@pytest.mark.parametrize("Sq", [1, 3])
def test_decode_appends_new_rows_in_place(Sq):
    """k_new / v_new are written into the caches at positions len - Sq + i, then attended."""
    cfg = DecodeConfig("append", 3, Sq, 2, 128, 2, 600, 128, True, seed=66 + Sq)
    q, kc, vc, table, lens = make_decode_inputs(cfg)
    g = torch.Generator().manual_seed(9)
    k_new = torch.randn((cfg.B, Sq, cfg.H, cfg.d), generator=g).to(torch.bfloat16)
    v_new = torch.randn((cfg.B, Sq, cfg.H, cfg.d), generator=g).to(torch.bfloat16)
    kc_d, vc_d = kc.cuda(), vc.cuda()
    o, lse = fa.attention_decode_paged(q.cuda(), kc_d, vc_d, table.cuda(), lens.cuda(), cfg.scale, True, (-1, -1), 0,
                                       k_new=k_new.cuda(), v_new=v_new.cuda())
    fa.check()
    o_ref, lse_ref = oracle_dec.decode_forward(q.double().numpy(), kc.double().numpy(), vc.double().numpy(),
                                               table.numpy(), lens.numpy(), cfg.scale, True,
                                               k_new=k_new.double().numpy(), v_new=v_new.double().numpy())
    assert_fwd_close(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref, f"append Sq={Sq}")
    # the caches now hold the new rows at their positions and are unchanged elsewhere
    k_exp = oracle_dec.append_rows(kc.double().numpy(), k_new.double().numpy(), table.numpy(), lens.numpy(),
                                   cfg.page_size)
    v_exp = oracle_dec.append_rows(vc.double().numpy(), v_new.double().numpy(), table.numpy(), lens.numpy(),
                                   cfg.page_size)
    assert np.array_equal(kc_d.double().cpu().numpy(), k_exp) and np.array_equal(vc_d.double().cpu().numpy(), v_exp)


def _expect_rows(o, lse, o_ref, lse_ref, seqlens, what):
    dead = ~np.isfinite(lse_ref)
    assert np.array_equal(dead, ~np.isfinite(lse)), f"{what}: rows without keys differ"
    if dead.any():
        assert (o[dead.transpose(0, 2, 1)] == 0).all()
    B, H = lse_ref.shape[:2]
    for b in range(B):
        for h in range(H):
            rows = np.nonzero(~dead[b, h])[0]
            if len(rows):
                assert_fwd_close(o[b, rows, h], lse[b, h, rows], o_ref[b, rows, h], lse_ref[b, h, rows],
                                 f"{what} b={b} h={h} len={int(seqlens[b])}")


@pytest.mark.parametrize("splits", [1, 5, 40])
@pytest.mark.parametrize("Sq,d,causal,win", [(8, 128, True, (-1, -1)), (2, 64, False, (3, 0)), (5, 128, True, (6, -1))])
def test_decode_append_across_splits(splits, Sq, d, causal, win):
    """Each new row is written by the split CTA whose key range holds it: rows that straddle a
    tile (and, with many splits, a split) boundary, sequences shorter than Sq, an empty one,
    window masks."""
    cfg = DecodeConfig("append_splits", 5, Sq, 3, d, 1, 700, 64, causal, seed=80 + Sq + splits)
    q, kc, vc, table, _ = make_decode_inputs(cfg)
    lens = torch.tensor([0, Sq - 1, 644, 64, 1], dtype=torch.int32)
    g = torch.Generator().manual_seed(90 + Sq)
    k_new = torch.randn((cfg.B, Sq, cfg.H, d), generator=g).to(torch.bfloat16)
    v_new = torch.randn((cfg.B, Sq, cfg.H, d), generator=g).to(torch.bfloat16)
    kc_d, vc_d = kc.cuda(), vc.cuda()
    o, lse = fa.attention_decode_paged(q.cuda(), kc_d, vc_d, table.cuda(), lens.cuda(), cfg.scale, causal, win, splits,
                                       k_new=k_new.cuda(), v_new=v_new.cuda())
    fa.check()
    o_ref, lse_ref = oracle_dec.decode_forward(q.double().numpy(), kc.double().numpy(), vc.double().numpy(),
                                               table.numpy(), lens.numpy(), cfg.scale, causal, *win,
                                               k_new=k_new.double().numpy(), v_new=v_new.double().numpy())
    _expect_rows(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref, lens,
                 f"append Sq={Sq} d={d} splits={splits}")
    for cache_d, cache, new in ((kc_d, kc, k_new), (vc_d, vc, v_new)):
        exp = oracle_dec.append_rows(cache.double().numpy(), new.double().numpy(), table.numpy(), lens.numpy(),
                                     cfg.page_size)
        assert np.array_equal(cache_d.double().cpu().numpy(), exp)


def test_decode_workspace_contents_do_not_matter():
    """The per-(b, h) arrival counters live in the caller's workspace and are zeroed by every
    call: a workspace filled with splits - 1 everywhere (a counter that would make the first
    arrival merge at once) and reused across calls gives the oracle's rows, bitwise the same
    every time (the merge sums the splits in a fixed order)."""
    cfg = DecodeConfig("workspace", 3, 2, 4, 128, 500, 1500, 128, True, seed=67)
    q, kc, vc, table, lens = (t.cuda() for t in make_decode_inputs(cfg))
    splits = 6
    nbytes = fa.decode_workspace_bytes(cfg.B, cfg.Sq, cfg.H, cfg.d, splits)
    assert nbytes > 0 and nbytes % 4 == 0
    ws = torch.full((nbytes // 4,), splits - 1, dtype=torch.int32, device="cuda").view(torch.uint8)
    o = torch.empty_like(q)
    lse = torch.empty((cfg.B, cfg.H, cfg.Sq), dtype=torch.float32, device="cuda")
    outs = []
    for _ in range(3):
        fa.decode_paged_into(q, kc, vc, table, lens, o, lse, cfg.scale, True, (-1, -1), splits, ws)
        fa.check()
        outs.append((o.clone(), lse.clone()))
    for o2, l2 in outs[1:]:
        assert torch.equal(o2, outs[0][0]) and torch.equal(l2, outs[0][1])
    o_ref, lse_ref = oracle_dec.decode_forward(q.cpu().double().numpy(), kc.cpu().double().numpy(),
                                               vc.cpu().double().numpy(), table.cpu().numpy(), lens.cpu().numpy(),
                                               cfg.scale, True)
    _expect_rows(outs[0][0].double().cpu().numpy(), outs[0][1].double().cpu().numpy(), o_ref, lse_ref,
                 lens.cpu(), "garbage workspace")


def test_decode_auto_pieces_fill_the_gpu_once():
    """fa_decode_splits: the automatic piece count lets all H x P CTAs run at once (no second
    wave) and leaves fewer than H SMs without a CTA (the tensor-core kernel for 4 or more rows
    takes a whole SM; H x P then falls short of the SM count by less than H); it never exceeds
    the batch's possible tiles."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for B, Sq, H, d, keys in [(8, 1, 16, 128, 8192), (8, 8, 16, 128, 8192), (4, 2, 8, 64, 4096), (1, 1, 2, 128, 65536)]:
        pieces = fa.decode_splits(B, Sq, H, d, keys)
        assert 1 <= pieces <= 65535
        assert pieces <= B * -(-keys // 64)
        assert H * pieces > sms - H, (B, Sq, H, d, pieces)  # all but fewer than H SMs busy
        assert H * pieces <= 8 * sms, (B, Sq, H, d, pieces)  # bounded by CTAs that fit per SM
    assert fa.decode_splits(1, 1, 2, 128, 64) == 1  # one tile: one piece
