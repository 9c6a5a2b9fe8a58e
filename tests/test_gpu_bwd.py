"""GPU parity of the backward pass (CUDA path through the C ABI) against the fp64 oracle.

The GPU backward consumes the GPU forward's O and LSE, as a training step does. Small and
ragged shapes are compared over whole tensors; the large workloads (the bench's launch
configuration) on whole sampled heads, plus identities that hold for every head.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_116_b200 as fa
from exact_attention_116_b200.inputs import CONFIGS, make_custom, make_inputs
from oracle import attention_fp64 as oracle
from parity import assert_bwd_close, to_np

pytestmark = pytest.mark.gpu


def gpu_fwd_bwd(q, k, v, do, scale, causal, win, workspace=None):
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.attention_fwd(qd, kd, vd, scale, causal, win)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, lse, dod, scale, causal, win, workspace=workspace)
    fa.check()
    return o, lse, dq, dk, dv


EDGE_CASES = [
    (1, 1, 1, 64, False, (-1, -1)),
    (1, 127, 2, 64, True, (-1, -1)),
    (2, 129, 1, 128, False, (-1, -1)),
    (1, 255, 2, 128, True, (-1, -1)),
    (1, 300, 2, 64, False, (5, 3)),
    (1, 513, 1, 128, False, (0, 0)),
    (1, 400, 1, 64, False, (1, 0)),
    (1, 384, 2, 128, True, (100, -1)),
    (1, 700, 2, 64, False, (128, 128)),
    (1, 600, 1, 128, False, (0, -1)),
    (2, 1000, 1, 128, False, (300, 17)),
    (1, 1030, 1, 64, True, (-1, -1)),
]


@pytest.mark.parametrize("B,N,H,d,causal,win", EDGE_CASES)
def test_bwd_edge_shapes(B, N, H, d, causal, win):
    q, k, v, do = make_custom(B, N, H, d, seed=2000 + N + d + 5 * H)
    scale = 1.0 / d ** 0.5
    _, _, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, scale, causal, win)
    ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), scale, causal, *win)
    assert_bwd_close([to_np(dq), to_np(dk), to_np(dv)], ref[:3], f"B{B} N{N} H{H} d{d} causal={causal} win={win}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("scale", [0.0, -0.3])
def test_bwd_scale_values(d, scale):
    q, k, v, do = make_custom(1, 260, 2, d, seed=91)
    for causal, win in [(False, (-1, -1)), (True, (-1, -1))]:
        _, _, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, scale, causal, win)
        ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), scale, causal, *win)
        # scale = 0 makes dQ and dK exactly zero in the oracle; compare them absolutely.
        if scale == 0.0:
            assert float(dq.abs().max()) == 0.0 and float(dk.abs().max()) == 0.0
            assert_bwd_close([to_np(dv)] * 3, [ref[2]] * 3, "scale=0 dV")
        else:
            assert_bwd_close([to_np(dq), to_np(dk), to_np(dv)], ref[:3], f"scale={scale} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_large_logits(d):
    q, k, v, do = make_custom(1, 640, 2, d, seed=17, qk_mult=8.0)
    for causal, win in [(False, (128, 128)), (True, (-1, -1))]:
        _, _, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, 1.0 / d ** 0.5, causal, win)
        ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), 1.0 / d ** 0.5, causal, *win)
        assert_bwd_close([to_np(dq), to_np(dk), to_np(dv)], ref[:3], f"x8 causal={causal} win={win}")


def test_bwd_workspace_paths_and_stages_agree():
    """Caller workspace, library-allocated workspace and the three staged calls give the same gradients."""
    B, N, H, d = 1, 500, 2, 128
    q, k, v, do = (x.cuda() for x in make_custom(B, N, H, d, seed=4))
    o, lse = fa.attention_fwd(q, k, v, None, True)
    ws = torch.empty(fa.workspace_bytes(B, N, H, d), dtype=torch.uint8, device="cuda")
    g1 = fa.attention_bwd(q, k, v, o, lse, do, None, True, workspace=ws)
    g2 = fa.attention_bwd(q, k, v, o, lse, do, None, True, workspace=None)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    fa.bwd_stages(q, k, v, o, lse, do, dq, dk, dv, ws, None, True)
    fa.check()
    for a, b in ((g1, g2), (g1, (dq, dk, dv))):
        assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])  # dK, dV: deterministic
        rel = float((a[0].float() - b[0].float()).norm() / b[0].float().norm())
        assert rel < 1e-3  # dQ: fp32 atomics may reorder additions


def _sampled_head_check(name, heads):
    cfg = CONFIGS[name]
    q, k, v, do = make_inputs(cfg)
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r))
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    # Identities for every head: sum_j dV_j = sum_i dO_i and sum_j dK_j = 0.
    sdv = dv.float().sum(dim=1)
    sdo = do.cuda().float().sum(dim=1)
    assert float((sdv - sdo).norm() / sdo.norm()) < 1e-2
    dkn = float(dk.float().norm())
    assert float(dk.float().sum(dim=1).norm()) < 1e-2 * dkn
    qn, kn, vn, don = (x.float().numpy() for x in (q, k, v, do))
    for b, h in heads:
        ref = oracle.head_backward(qn[b, :, h].astype(np.float64), kn[b, :, h].astype(np.float64),
                                   vn[b, :, h].astype(np.float64), don[b, :, h].astype(np.float64), cfg.scale,
                                   cfg.causal, cfg.win_l, cfg.win_r, block_rows=1024)
        got = [to_np(t[b, :, h]) for t in (dq, dk, dv)]
        assert_bwd_close(got, ref[:3], f"{name} head {(b, h)}")


def test_bwd_train_config_sampled_heads():
    _sampled_head_check("train_fwd_bwd", [(0, 0), (1, 15)])


def test_bwd_window_config_sampled_heads():
    _sampled_head_check("window_fwd_bwd", [(0, 0), (1, 15), (1, 4)])


def test_bwd_long_config_sampled_head():
    _sampled_head_check("long_fwd_bwd", [(0, 9)])


def test_autograd_matches_explicit_calls():
    q, k, v, do = (x.cuda() for x in make_custom(1, 300, 2, 64, seed=8))
    qr, kr, vr = (x.clone().requires_grad_(True) for x in (q, k, v))
    o = fa.flash_attention(qr, kr, vr, None, True)
    o.backward(do)
    o2, lse = fa.attention_fwd(q, k, v, None, True)
    g = fa.attention_bwd(q, k, v, o2, lse, do, None, True)
    assert torch.equal(kr.grad, g[1]) and torch.equal(vr.grad, g[2])
    assert float((qr.grad.float() - g[0].float()).norm() / g[0].float().norm()) < 1e-3
