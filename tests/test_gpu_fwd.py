"""GPU parity of the forward pass (CUDA path through the C ABI) against the fp64 oracle.

Small and ragged shapes and the GPT-style workload are compared element by element over whole
tensors; the large workloads run in the same launch configuration the bench uses and are
compared over every row of sampled heads.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_116_b200 as fa
from exact_attention_116_b200.inputs import CONFIGS, make_custom, make_inputs
from oracle import attention_fp64 as oracle
from parity import assert_fwd_close, to_np

pytestmark = pytest.mark.gpu


def gpu_fwd(q, k, v, scale, causal, win):
    o, lse = fa.attention_fwd(q.cuda(), k.cuda(), v.cuda(), scale, causal, win)
    fa.check()
    return o, lse


EDGE_CASES = [
    # B, N, H, d, causal, window
    (1, 1, 1, 64, False, (-1, -1)),
    (1, 1, 2, 128, True, (-1, -1)),
    (1, 127, 2, 64, True, (-1, -1)),
    (2, 129, 1, 128, False, (-1, -1)),
    (1, 100, 2, 128, False, (-1, -1)),
    (1, 255, 3, 128, True, (-1, -1)),
    (1, 256, 2, 64, False, (-1, -1)),
    (1, 300, 2, 64, False, (5, 3)),
    (1, 513, 1, 128, False, (0, 0)),
    (1, 400, 2, 64, False, (1, 0)),
    (1, 384, 1, 128, True, (100, -1)),
    (1, 700, 2, 64, False, (128, 128)),
    (1, 600, 1, 128, False, (0, -1)),
    (2, 1000, 2, 128, False, (300, 17)),
    (1, 1030, 1, 64, True, (-1, -1)),
    (1, 640, 2, 128, False, (-1, 200)),
]


@pytest.mark.parametrize("B,N,H,d,causal,win", EDGE_CASES)
def test_fwd_edge_shapes(B, N, H, d, causal, win):
    q, k, v, _ = make_custom(B, N, H, d, seed=1000 + N + d + 7 * H)
    scale = 1.0 / d ** 0.5
    o, lse = gpu_fwd(q, k, v, scale, causal, win)
    o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), scale, causal, *win)
    assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, f"B{B} N{N} H{H} d{d} causal={causal} win={win}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("scale", [0.0, -0.2, 0.9])
def test_fwd_scale_values(d, scale):
    q, k, v, _ = make_custom(1, 300, 2, d, seed=77)
    for causal, win in [(False, (-1, -1)), (True, (-1, -1)), (False, (20, 9))]:
        o, lse = gpu_fwd(q, k, v, scale, causal, win)
        o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), scale, causal, *win)
        assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, f"scale={scale} causal={causal} win={win}")


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_large_logits(d):
    """Q and K scaled by 8: logits of a few hundred exercise the running-max rescaling."""
    q, k, v, _ = make_custom(1, 777, 2, d, seed=5, qk_mult=8.0)
    for causal, win in [(False, (-1, -1)), (True, (-1, -1)), (False, (128, 128))]:
        o, lse = gpu_fwd(q, k, v, 1.0 / d ** 0.5, causal, win)
        o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), 1.0 / d ** 0.5, causal, *win)
        assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, f"x8 causal={causal} win={win}")


def test_fwd_tiny_config_full():
    cfg = CONFIGS["tiny_fwd"]
    q, k, v, _ = make_inputs(cfg)
    o, lse = gpu_fwd(q, k, v, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r))
    o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), cfg.scale, cfg.causal, cfg.win_l,
                                              cfg.win_r)
    assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, "tiny_fwd")


def test_fwd_gpt_config_full_and_determinism():
    """The GPT-style workload (B4 H16 N2048 d64 causal) against the oracle over all 64 heads, element
    by element, and bitwise equal across two calls."""
    cfg = CONFIGS["gpt_fwd"]
    q, k, v, _ = make_inputs(cfg)
    o, lse = gpu_fwd(q, k, v, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r))
    o2, lse2 = gpu_fwd(q, k, v, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r))
    assert torch.equal(o, o2) and torch.equal(lse, lse2), "forward is not bitwise reproducible"
    o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), cfg.scale, cfg.causal, cfg.win_l,
                                              cfg.win_r)
    assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, "gpt_fwd (all heads)")


@pytest.mark.parametrize("name", ["train_fwd_bwd", "long_fwd_bwd", "window_fwd_bwd"])
def test_fwd_full_size_whole_heads(name):
    """The large workloads in the bench's launch configuration: every row of three heads, the first,
    the last and one drawn at random (heads are independent, so each comparison is exact for its head),
    and finite outputs everywhere."""
    cfg = CONFIGS[name]
    q, k, v, _ = make_inputs(cfg)
    o, lse = gpu_fwd(q, k, v, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r))
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(sum(map(ord, name)))
    heads = [(0, 0), (cfg.B - 1, cfg.H - 1), (int(rng.integers(cfg.B)), int(rng.integers(cfg.H)))]
    on, ln_ = to_np(o), to_np(lse)
    qn, kn, vn = (x.float().numpy() for x in (q, k, v))
    for b, h in heads:
        o_ref, lse_ref = oracle.head_forward(qn[b, :, h].astype(np.float64), kn[b, :, h].astype(np.float64),
                                             vn[b, :, h].astype(np.float64), cfg.scale, cfg.causal, cfg.win_l,
                                             cfg.win_r, block_rows=1024)
        assert_fwd_close(on[b, :, h], ln_[b, h], o_ref, lse_ref, f"{name} head {(b, h)}")


def test_fwd_autograd_wrapper_matches():
    q, k, v, _ = make_custom(1, 200, 2, 64, seed=3)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o1 = fa.flash_attention(qd, kd, vd, None, True)
    o2, _ = fa.attention_fwd(qd, kd, vd, None, True)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,N,H", [(2, 777, 48), (3, 200, 64)])
def test_fwd_many_items_per_cta(d, B, N, H):
    """More work items than SMs, so each CTA runs several items back to back: the next item's
    Q and K/V loads and its first scores overlap the previous item's last tiles and epilogue."""
    q, k, v, _ = make_custom(B, N, H, d, seed=600 + N + d)
    for causal, win in [(True, (-1, -1)), (False, (64, 200)), (False, (-1, -1))]:
        o, lse = gpu_fwd(q, k, v, None, causal, win)
        o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), 1.0 / d ** 0.5, causal, *win)
        assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, f"B{B} N{N} H{H} d{d} causal={causal} win={win}")
