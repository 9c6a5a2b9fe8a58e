"""GPU parity of ALiBi attention (fa_fwd_ex / fa_bwd_ex, through the C ABI) against the fp64 oracle.

The slopes are per (batch, head): the usual geometric sequence 2^(-8(h+1)/H), scaled per batch
so that the two batches differ. Tolerances are those of the bf16 path (forward
max |ΔO| / max(1, |O|) <= 1e-2, max |ΔLSE| <= 1e-3; backward relative L2 <= 1e-2 per
gradient); both backward algorithms (fp32 dQ accumulation and the deterministic dQ pass) are
checked.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_116_b200 as fa
from exact_attention_116_b200.inputs import make_custom
from oracle import attention_fp64 as oracle
from parity import assert_bwd_close, assert_fwd_close, to_np

pytestmark = pytest.mark.gpu


def slopes_for(B, H, spread=1.0):
    base = np.array([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)])
    return np.stack([base * spread * (1.0 + 0.5 * b) for b in range(B)]).astype(np.float32)


def run(B, N, H, d, causal, win, seed, spread=1.0, deterministic=False, scale=None):
    q, k, v, do = make_custom(B, N, H, d, seed=seed)
    sl = slopes_for(B, H, spread)
    sl_d = torch.from_numpy(sl).cuda()
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.attention_fwd(qd, kd, vd, scale, causal, win, alibi_slopes=sl_d)
    g = fa.attention_bwd(qd, kd, vd, o, lse, dod, scale, causal, win, deterministic=deterministic,
                         alibi_slopes=sl_d)
    fa.check()
    return (q, k, v, do), sl, (o, lse), g


EDGE = [
    (1, 1, 1, 64, False, (-1, -1)),
    (1, 127, 2, 64, True, (-1, -1)),
    (2, 129, 2, 128, False, (-1, -1)),
    (1, 300, 2, 64, False, (5, 3)),
    (1, 384, 2, 128, True, (100, -1)),
    (2, 700, 2, 64, False, (128, 128)),
    (1, 1030, 2, 128, True, (-1, -1)),
]


@pytest.mark.parametrize("deterministic", [False, True])
@pytest.mark.parametrize("B,N,H,d,causal,win", EDGE)
def test_alibi_fwd_bwd_edge_shapes(B, N, H, d, causal, win, deterministic):
    (q, k, v, do), sl, (o, lse), g = run(B, N, H, d, causal, win, seed=5000 + N + d, deterministic=deterministic)
    scale = 1.0 / d ** 0.5
    o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), scale, causal, *win, alibi_slopes=sl)
    assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, f"alibi fwd B{B} N{N} d{d} causal={causal} win={win}")
    ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), scale, causal, *win, alibi_slopes=sl)
    assert_bwd_close([to_np(t) for t in g], ref[:3], f"alibi bwd det={deterministic} B{B} N{N} d{d}")


@pytest.mark.parametrize("d", [64, 128])
def test_alibi_steep_and_negative_scale(d):
    """Steep slopes (most weight on the nearest keys) and a negative softmax scale."""
    for spread, scale in ((16.0, None), (1.0, -0.2)):
        (q, k, v, do), sl, (o, lse), g = run(2, 500, 2, d, False, (-1, -1), seed=91 + d, spread=spread, scale=scale)
        sc = 1.0 / d ** 0.5 if scale is None else scale
        o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), sc, False, alibi_slopes=sl)
        assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, f"alibi spread={spread} scale={sc}")
        ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), sc, False, alibi_slopes=sl)
        assert_bwd_close([to_np(t) for t in g], ref[:3], f"alibi bwd spread={spread} scale={sc}")


def test_alibi_zero_slopes_match_plain_path():
    q, k, v, do = (x.cuda() for x in make_custom(1, 400, 2, 128, seed=92))
    zero = torch.zeros((1, 2), dtype=torch.float32, device="cuda")
    o0, l0 = fa.attention_fwd(q, k, v, None, True)
    o1, l1 = fa.attention_fwd(q, k, v, None, True, alibi_slopes=zero)
    g0 = fa.attention_bwd(q, k, v, o0, l0, do, None, True)
    g1 = fa.attention_bwd(q, k, v, o1, l1, do, None, True, alibi_slopes=zero)
    fa.check()
    assert float((o0.float() - o1.float()).abs().max()) < 1e-2 and float((l0 - l1).abs().max()) < 1e-4
    for a, b in zip(g0, g1):
        assert float((a.float() - b.float()).norm() / b.float().norm()) < 1e-2


def test_alibi_long_causal_sampled_heads():
    B, N, H, d = 1, 4096, 8, 128
    (q, k, v, do), sl, (o, lse), g = run(B, N, H, d, True, (-1, -1), seed=93)
    qn, kn, vn, don = (x.double().numpy() for x in (q, k, v, do))
    for h in (0, 7):
        o_ref, lse_ref = oracle.head_forward(qn[0, :, h], kn[0, :, h], vn[0, :, h], 1 / d ** 0.5, True,
                                             block_rows=1024, alibi=float(sl[0, h]))
        assert_fwd_close(to_np(o[0, :, h]), to_np(lse[0, h]), o_ref, lse_ref, f"alibi long head {h}")
        ref = oracle.head_backward(qn[0, :, h], kn[0, :, h], vn[0, :, h], don[0, :, h], 1 / d ** 0.5, True,
                                   block_rows=1024, alibi=float(sl[0, h]))
        assert_bwd_close([to_np(t[0, :, h]) for t in g], ref[:3], f"alibi long head {h}")
