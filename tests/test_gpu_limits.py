"""GPU parity at the size limits: the longest sequence, the most heads, the longest KV cache.

* N = 131072 tokens (one head, causal): forward rows sampled at both ends and in the middle;
  backward checked exactly where the oracle can afford it — under causal masking the last 256
  keys are seen only by the last 256 queries, so backward_rows on those queries gives the
  exact dK, dV of those keys and dQ of those queries; the first 128 queries see only the first
  128 keys — plus the identities sum_j dV_j = sum_i dO_i and sum_j dK_j = 0 over the whole head.
* B x H = 512 heads of 200 tokens (far more work items than SMs), compared over whole tensors.
* A paged decode against one 65536-key sequence.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_116_b200 as fa
from exact_attention_116_b200.inputs import DecodeConfig, make_custom, make_decode_inputs
from oracle import attention_fp64 as oracle
from oracle import decode_paged_fp64 as oracle_dec
from parity import assert_bwd_close, assert_fwd_close, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
def test_longest_sequence(d):
    N = 131072
    q, k, v, do = make_custom(1, N, 1, d, seed=700 + d)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    scale = d ** -0.5
    o, lse = fa.attention_fwd(qd, kd, vd, scale, True)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, lse, dod, scale, True)
    fa.check()
    qn, kn, vn, don = (x.double().numpy() for x in (q, k, v, do))
    rows = [0, 1, 127, 128, 4095, N // 2, N - 129, N - 1]
    o_ref, lse_ref = oracle.forward_rows(qn, kn, vn, 0, 0, rows, scale, True)
    assert_fwd_close(to_np(o[0, rows, 0]), to_np(lse[0, 0, rows]), o_ref, lse_ref, f"N={N} d={d} forward rows")
    # identities over the whole head
    sdv, sdo = dv.double().sum(dim=1), do.double().sum(dim=1)
    assert float((sdv.cpu() - sdo).norm() / sdo.norm()) < 1e-2
    assert float(dk.double().sum(dim=1).norm()) < 1e-2 * float(dk.double().norm())
    h = (qn[0, :, 0], kn[0, :, 0], vn[0, :, 0], don[0, :, 0])
    for r0, r1 in ((N - 256, N), (0, 128)):
        dq_r = np.zeros((N, d))
        dk_r = np.zeros((N, d))
        dv_r = np.zeros((N, d))
        dvec = np.zeros(N)
        oracle.backward_rows(*h, r0, r1, scale, True, -1, -1, dq_r, dk_r, dv_r, dvec)
        got_q = to_np(dq[0, r0:r1, 0])
        floor = 1e-3 * float(np.linalg.norm(dv_r[r0:r1]))
        e = float(np.linalg.norm(got_q - dq_r[r0:r1]) / max(np.linalg.norm(dq_r[r0:r1]), floor))
        assert e <= 1e-2, f"dQ rows [{r0},{r1}): {e:.3e}"
        if r0 == N - 256:  # the last keys: these queries are their only ones
            assert_bwd_close([got_q, to_np(dk[0, r0:r1, 0]), to_np(dv[0, r0:r1, 0])],
                             [dq_r[r0:r1], dk_r[r0:r1], dv_r[r0:r1]], f"N={N} last 256 keys")


def test_many_heads():
    B, N, H, d = 8, 200, 64, 128
    q, k, v, do = make_custom(B, N, H, d, seed=710)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.attention_fwd(qd, kd, vd, None, False, (40, 60))
    g = fa.attention_bwd(qd, kd, vd, o, lse, dod, None, False, (40, 60))
    fa.check()
    o_ref, lse_ref = oracle.attention_forward(to_np(q), to_np(k), to_np(v), d ** -0.5, False, 40, 60)
    assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, "512 heads forward")
    ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), d ** -0.5, False, 40, 60)
    for name, got, r in zip(("dQ", "dK", "dV"), g, ref[:3]):
        assert rel_l2(to_np(got), r) <= 1e-2, name


def test_longest_kv_cache():
    cfg = DecodeConfig("long_cache", 1, 2, 2, 128, 65536, 65536, 256, True, seed=720)
    host = make_decode_inputs(cfg)
    o, lse = fa.attention_decode_paged(*(t.cuda() for t in host), cfg.scale, True, (-1, -1), 0)
    fa.check()
    q, kc, vc, table, lens = host
    o_ref, lse_ref = oracle_dec.decode_forward(q.double().numpy(), kc.float().numpy(), vc.float().numpy(),
                                               table.numpy(), lens.numpy(), cfg.scale, True)
    assert_fwd_close(to_np(o), to_np(lse), o_ref, lse_ref, "65536-key decode")
