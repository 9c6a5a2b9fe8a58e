"""GPU parity of packed variable-length batches (fa_fwd_varlen / fa_bwd_varlen) against the oracle.

The sequences are packed along the token axis and attended on their own. Tolerances are those
of the bf16 path. Lengths include empty sequences, single tokens and lengths around the
128-row tile, so that tiles straddle sequence boundaries; both backward algorithms and ALiBi
are covered.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_116_b200 as fa
from oracle import varlen_fp64 as oracle_vl
from parity import assert_bwd_close, assert_fwd_close, to_np

pytestmark = pytest.mark.gpu


def packed_inputs(lens, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    total = int(sum(lens))
    xs = [torch.randn((total, H, d), generator=g).to(torch.bfloat16) for _ in range(4)]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return xs, cu


def run(lens, H, d, causal, win, seed, deterministic=False, slopes=None):
    (q, k, v, do), cu = packed_inputs(lens, H, d, seed)
    dev = [x.cuda() for x in (q, k, v, do)]
    cu_d = cu.cuda()
    sl = None if slopes is None else torch.tensor(slopes, dtype=torch.float32).cuda()
    o, lse = fa.attention_fwd_varlen(dev[0], dev[1], dev[2], cu_d, None, causal, win, alibi_slopes=sl)
    g = fa.attention_bwd_varlen(dev[0], dev[1], dev[2], o, lse, dev[3], cu_d, None, causal, win,
                                deterministic=deterministic, alibi_slopes=sl)
    fa.check()
    return (q, k, v, do), cu, (o, lse), g


def compare(inputs, cu, out, g, d, causal, win, what, slopes=None, rows=None):
    q, k, v, do = (to_np(x) for x in inputs)
    scale = 1.0 / d ** 0.5
    o_ref, lse_ref = oracle_vl.varlen_forward(q, k, v, cu.numpy(), scale, causal, *win, alibi_slopes=slopes)
    o, lse = to_np(out[0]), to_np(out[1])
    live = np.isfinite(lse_ref)  # tokens of empty sequences do not exist; every other row sees a key
    assert live.all()
    assert_fwd_close(o, lse.T, o_ref, lse_ref.T, f"{what} forward")
    ref = oracle_vl.varlen_backward(q, k, v, do, cu.numpy(), scale, causal, *win, alibi_slopes=slopes)
    assert_bwd_close([to_np(t) for t in g], ref, f"{what} backward")


LENS = [[300], [1, 0, 129, 128, 127, 5], [700, 1, 250, 0, 513], [64] * 9]


@pytest.mark.parametrize("deterministic", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("lens", LENS, ids=lambda x: f"{len(x)}seq")
def test_varlen_causal(lens, d, deterministic):
    inputs, cu, out, g = run(lens, 2, d, True, (-1, -1), seed=sum(lens) + d, deterministic=deterministic)
    compare(inputs, cu, out, g, d, True, (-1, -1), f"lens={lens} d={d} det={deterministic}")


@pytest.mark.parametrize("causal,win", [(False, (-1, -1)), (False, (40, 7)), (True, (100, -1))])
def test_varlen_masks(causal, win):
    lens = [200, 3, 0, 400, 129]
    inputs, cu, out, g = run(lens, 3, 128, causal, win, seed=77)
    compare(inputs, cu, out, g, 128, causal, win, f"causal={causal} win={win}")


def test_varlen_with_alibi():
    lens = [150, 300, 1, 260]
    slopes = [0.5, 0.0625, 0.01]
    inputs, cu, out, g = run(lens, 3, 64, True, (-1, -1), seed=78, slopes=slopes)
    compare(inputs, cu, out, g, 64, True, (-1, -1), "alibi", slopes=np.asarray(slopes))


def test_varlen_training_mix_sampled_sequences():
    """A training-like batch: 8 sequences of 512..4096 tokens (16K tokens, H16 d128, causal)."""
    lens = [4096, 512, 3000, 1024, 2048, 777, 2500, 2427]
    (q, k, v, do), cu = packed_inputs(lens, 16, 128, 79)
    dev = [x.cuda() for x in (q, k, v, do)]
    o, lse = fa.attention_fwd_varlen(dev[0], dev[1], dev[2], cu.cuda(), None, True)
    g = fa.attention_bwd_varlen(dev[0], dev[1], dev[2], o, lse, dev[3], cu.cuda(), None, True)
    fa.check()
    for b in (1, 5, 7):  # whole sequences, heads 0 and 15
        t0, t1 = int(cu[b]), int(cu[b + 1])
        sub = [to_np(x[t0:t1])[:, [0, 15]] for x in (q, k, v, do)]
        cu_b = np.array([0, t1 - t0])
        o_ref, lse_ref = oracle_vl.varlen_forward(*sub[:3], cu_b, 128 ** -0.5, True)
        assert_fwd_close(to_np(o[t0:t1])[:, [0, 15]], to_np(lse[[0, 15], t0:t1]).T, o_ref, lse_ref.T, f"mix seq {b}")
        ref = oracle_vl.varlen_backward(*sub, cu_b, 128 ** -0.5, True)
        assert_bwd_close([to_np(t[t0:t1])[:, [0, 15]] for t in g], ref, f"mix seq {b}")


def test_varlen_bad_offsets_are_reported_not_followed():
    (q, k, v, _), cu = packed_inputs([100, 60], 2, 64, 80)
    bad = torch.tensor([0, 100, 150], dtype=torch.int32).cuda()  # ends before total = 160
    o, lse = fa.attention_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), bad, None, True)
    with pytest.raises(fa.FaError) as e:
        fa.check()
    assert e.value.status == 6  # FA_ERR_DEVICE
    assert torch.isfinite(o[:150].float()).all()
    fa.check()  # cleared; the context is usable


def test_varlen_forward_is_bitwise_reproducible_and_ordered_by_cost():
    """Many sequences of mixed lengths, so that the cost-sorted pair order differs from the index
    order: two calls give the same bits, and rows match the oracle."""
    lens = [900, 3, 0, 1500, 77, 640, 256, 1, 1100, 300, 2049, 128]
    (q, k, v, do), cu = packed_inputs(lens, 2, 128, seed=91)
    dev = [x.cuda() for x in (q, k, v)]
    cu_d = cu.cuda()
    o1, l1 = fa.attention_fwd_varlen(*dev, cu_d, None, True)
    o2, l2 = fa.attention_fwd_varlen(*dev, cu_d, None, True)
    fa.check()
    assert torch.equal(o1, o2) and torch.equal(l1, l2), "packed forward is not bitwise reproducible"
    o_ref, lse_ref = oracle_vl.varlen_forward(to_np(q), to_np(k), to_np(v), cu.numpy(), 128 ** -0.5, True, -1, -1)
    assert_fwd_close(to_np(o1), to_np(l1).T, o_ref, lse_ref.T, "mixed packed forward")
