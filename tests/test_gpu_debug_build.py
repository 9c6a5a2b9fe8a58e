"""The bounds-checking build of the library (libfa_sm100_debug.so, compiled with -DFA_DEBUG=1).

A memory checker cannot be run on these GPUs, so the kernels carry their own: in this build
every computed TMA coordinate (and its 16-byte alignment), bulk-copy range, shared-memory
destination and global index is checked on the device before it is used, and a failed check
is reported through fa_check (FA_ERR_DEVICE) instead of touching memory out of range. These
tests run the edge-shape suites of every entry point through that build and require both
oracle parity and fa_check() == FA_OK after every call, i.e. no check ever fires.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_116_b200 as fa
from exact_attention_116_b200 import binding
from exact_attention_116_b200 import build as cuda_build
from exact_attention_116_b200.inputs import AttnConfig, DecodeConfig, make_custom, make_decode_inputs, make_fp8_inputs
from oracle import attention_fp64 as oracle
from oracle import decode_paged_fp64 as oracle_dec
from oracle import fp8_e4m3 as oracle8
from oracle import varlen_fp64 as oracle_vl
from parity import assert_bwd_close, assert_fwd_close, to_np
from test_gpu_bwd import EDGE_CASES as BWD_EDGE_CASES
from test_gpu_fwd import EDGE_CASES as FWD_EDGE_CASES

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def debug_lib():
    return binding.open_library(cuda_build.build(debug=True))


@pytest.fixture(autouse=True)
def use_debug_lib(debug_lib, monkeypatch):
    """Route every wrapper (and fa.check) to the bounds-checking build for the test."""
    monkeypatch.setattr(binding, "_lib", debug_lib)
    yield


def test_the_debug_build_is_the_one_called(debug_lib):
    assert binding.load() is debug_lib
    assert debug_lib._name.endswith("libfa_sm100_debug.so")


@pytest.mark.parametrize("B,N,H,d,causal,win", FWD_EDGE_CASES)
def test_debug_build_forward_edge_shapes(B, N, H, d, causal, win):
    q, k, v, _ = make_custom(B, N, H, d, seed=1000 + N + d + 7 * H)
    o, lse = fa.attention_fwd(q.cuda(), k.cuda(), v.cuda(), None, causal, win)
    fa.check()
    o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), d ** -0.5, causal, *win)
    assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, f"debug build B{B} N{N} H{H} d{d} {causal} {win}")


@pytest.mark.parametrize("deterministic", [False, True])
@pytest.mark.parametrize("B,N,H,d,causal,win", BWD_EDGE_CASES)
def test_debug_build_backward_edge_shapes(B, N, H, d, causal, win, deterministic):
    q, k, v, do = (x.cuda() for x in make_custom(B, N, H, d, seed=2000 + N + d + 5 * H))
    o, lse = fa.attention_fwd(q, k, v, None, causal, win)
    g = fa.attention_bwd(q, k, v, o, lse, do, None, causal, win, deterministic=deterministic)
    fa.check()
    ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), d ** -0.5, causal, *win)
    assert_bwd_close([to_np(t) for t in g], ref[:3], f"debug build B{B} N{N} H{H} d{d} {causal} {win}")


def test_debug_build_alibi_staged_and_static_workspace():
    B, N, H, d = 2, 300, 3, 64
    q, k, v, do = (x.cuda() for x in make_custom(B, N, H, d, seed=31))
    slopes = torch.tensor([[0.5, 0.1, 0.02], [0.25, 0.05, 0.0]], dtype=torch.float32).cuda()
    o, lse = fa.attention_fwd(q, k, v, None, True, (-1, -1), alibi_slopes=slopes)
    g = fa.attention_bwd(q, k, v, o, lse, do, None, True, (-1, -1), alibi_slopes=slopes)
    fa.check()
    o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), d ** -0.5, True,
                                              alibi_slopes=slopes.cpu().numpy())
    assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, "debug build alibi forward")
    ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), d ** -0.5, True,
                                    alibi_slopes=slopes.cpu().numpy())
    assert_bwd_close([to_np(t) for t in g], ref[:3], "debug build alibi backward")
    o, lse = fa.attention_fwd(q, k, v, None, False, (20, 7))
    ws = torch.empty(fa.workspace_bytes(B, N, H, d), dtype=torch.uint8, device="cuda")
    staged = [torch.empty_like(q) for _ in range(3)]
    fa.bwd_stages(q, k, v, o, lse, do, *staged, ws, None, False, (20, 7))
    fixed = [torch.empty_like(q) for _ in range(3)]
    binding.bwd_into_static_workspace(q, k, v, o, lse, do, *fixed, None, False, (20, 7))
    fa.check()
    ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), d ** -0.5, False, 20, 7)
    assert_bwd_close([to_np(t) for t in staged], ref[:3], "debug build staged backward")
    assert_bwd_close([to_np(t) for t in fixed], ref[:3], "debug build allocation-free backward")


@pytest.mark.parametrize("lens", [[200, 3, 0, 400, 129], [1, 1, 700], [257, 1000, 64]])
def test_debug_build_packed_batches(lens):
    H, d = 2, 128
    total = sum(lens)
    q, k, v, do = make_custom(1, total, H, d, seed=41 + total)
    q, k, v, do = (x[0] for x in (q, k, v, do))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    dev = [x.cuda() for x in (q, k, v, do)]
    o, lse = fa.attention_fwd_varlen(dev[0], dev[1], dev[2], cu.cuda(), None, True)
    g = fa.attention_bwd_varlen(dev[0], dev[1], dev[2], o, lse, dev[3], cu.cuda(), None, True)
    fa.check()
    o_ref, lse_ref = oracle_vl.varlen_forward(to_np(q), to_np(k), to_np(v), cu.numpy(), d ** -0.5, True, -1, -1)
    assert_fwd_close(to_np(o), to_np(lse).T, o_ref, lse_ref.T, f"debug build packed {lens}")
    ref = oracle_vl.varlen_backward(to_np(q), to_np(k), to_np(v), to_np(do), cu.numpy(), d ** -0.5, True)
    assert_bwd_close([to_np(t) for t in g], ref, f"debug build packed {lens}")


@pytest.mark.parametrize("N,causal,win", [(200, True, (-1, -1)), (333, False, (50, 20)), (1, False, (-1, -1))])
def test_debug_build_fp8_forward(N, causal, win):
    cfg = AttnConfig("dbg_fp8", 1, N, 2, 128, causal, win[0], win[1], seed=50 + N)
    codes, desc = make_fp8_inputs(cfg)
    o, lse = fa.attention_fwd_fp8(*(t.cuda() for t in (*codes, *desc)), cfg.scale, causal, win)
    fa.check()
    cn, dn = [t.numpy() for t in codes], [t.numpy().astype(np.float64) for t in desc]
    o_ref, lse_ref = oracle8.attention_forward_fp8(*cn, *dn, cfg.scale, causal, *win)
    vmax = np.abs(oracle8.dequantize(cn[2], dn[2])).max()
    assert float(np.abs(o.double().cpu().numpy() - o_ref).max()) <= 2.0 ** -4 * vmax
    assert float(np.abs(lse.double().cpu().numpy() - lse_ref).max()) <= 1e-3


@pytest.mark.parametrize("Sq,splits,append", [(1, 0, False), (2, 3, True), (4, 1, True), (7, 0, False)])
def test_debug_build_paged_decode(Sq, splits, append):
    cfg = DecodeConfig("dbg_decode", 5, Sq, 2, 128, 1, 700, 128, True, seed=60 + Sq)
    q, kc, vc, table, lens = make_decode_inputs(cfg)
    lens = torch.tensor([700, 0, 1, 129, 300], dtype=torch.int32)
    kwargs = {}
    if append:  # new rows equal to the cache rows they overwrite: the cache stays as generated
        k_new, v_new = torch.empty_like(q), torch.empty_like(q)
        for b in range(cfg.B):
            for i in range(Sq):
                pos = int(lens[b]) - Sq + i
                if pos < 0:
                    continue
                page = int(table[b, pos // cfg.page_size])
                k_new[b, i], v_new[b, i] = kc[page, pos % cfg.page_size], vc[page, pos % cfg.page_size]
        kwargs = {"k_new": k_new.cuda(), "v_new": v_new.cuda()}
    o, lse = fa.attention_decode_paged(*(t.cuda() for t in (q, kc, vc, table, lens)), cfg.scale, True, (-1, -1),
                                       splits, **kwargs)
    fa.check()
    o_ref, lse_ref = oracle_dec.decode_forward(q.double().numpy(), kc.double().numpy(), vc.double().numpy(),
                                               table.numpy(), lens.numpy(), cfg.scale, True)
    on, ln_ = o.double().cpu().numpy(), lse.double().cpu().numpy()
    for b in range(cfg.B):
        for h in range(cfg.H):
            rows = np.nonzero(np.isfinite(lse_ref[b, h]))[0]
            assert (~np.isfinite(ln_[b, h]) == ~np.isfinite(lse_ref[b, h])).all()
            if len(rows):
                assert_fwd_close(on[b, rows, h], ln_[b, h, rows], o_ref[b, rows, h], lse_ref[b, h, rows],
                                 f"debug build decode Sq={Sq} b={b} h={h}")
