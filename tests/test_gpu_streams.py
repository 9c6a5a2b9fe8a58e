"""Concurrent calls on several CUDA streams (GPU).

Each forward call takes its own slot of the library's work-counter ring and each backward call
uses its own workspace, so calls that overlap on the GPU must not disturb one another: every
result equals the same call made alone. The forward computes each work item in one CTA,
whichever CTA takes it, so O and LSE are compared bit for bit; so are dK and dV (each KV tile's
sums are formed in one CTA in a fixed order). dQ is a sum of partial products added in the
order the CTAs finish, so it is compared within a few bf16 ulps.
"""

from __future__ import annotations

import pytest
import torch

import exact_attention_116_b200 as fa
from exact_attention_116_b200 import binding
from exact_attention_116_b200.inputs import AttnConfig, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    AttnConfig("s0", 2, 4096, 8, 128, True, seed=301),
    AttnConfig("s1", 1, 8192, 4, 64, False, 128, 128, seed=302),
    AttnConfig("s2", 3, 1000, 6, 128, False, seed=303),
    AttnConfig("s3", 2, 2048, 16, 64, True, 256, -1, seed=304),
]


def _inputs(cfg):
    return [x.cuda() for x in make_inputs(cfg)]


def test_fwd_concurrent_streams_match_single_calls():
    dev = torch.device("cuda", 0)
    data = [_inputs(c) for c in CASES]
    ref = []
    for cfg, (q, k, v, _) in zip(CASES, data):
        o, lse = fa.attention_fwd(q, k, v, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r))
        ref.append((o, lse))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(device=dev) for _ in CASES]
    outs = [[(torch.empty_like(q), torch.empty(q.shape[0], q.shape[2], q.shape[1], device=dev))
             for _ in range(3)] for (q, _, _, _) in data]
    for rnd in range(3):  # three rounds, each call on its own stream, none waiting for another
        for s, cfg, (q, k, v, _), buf in zip(streams, CASES, data, outs):
            with torch.cuda.stream(s):
                binding.fwd_into(q, k, v, buf[rnd][0], buf[rnd][1], cfg.scale, cfg.causal,
                                 (cfg.win_l, cfg.win_r), stream=s)
    torch.cuda.synchronize()
    fa.check()
    for cfg, (o_ref, lse_ref), buf in zip(CASES, ref, outs):
        for rnd, (o, lse) in enumerate(buf):
            assert torch.equal(o, o_ref), f"{cfg.name} round {rnd}: O differs"
            assert torch.equal(lse, lse_ref), f"{cfg.name} round {rnd}: LSE differs"


def test_bwd_concurrent_streams_match_single_calls():
    dev = torch.device("cuda", 0)
    data = [_inputs(c) for c in CASES]
    fwd, ref = [], []
    for cfg, (q, k, v, do) in zip(CASES, data):
        win = (cfg.win_l, cfg.win_r)
        o, lse = fa.attention_fwd(q, k, v, cfg.scale, cfg.causal, win)
        fwd.append((o, lse))
        ref.append(fa.attention_bwd(q, k, v, o, lse, do, cfg.scale, cfg.causal, win))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(device=dev) for _ in CASES]
    grads, works = [], []
    for cfg, (q, _, _, _) in zip(CASES, data):
        B, N, H, d = q.shape
        grads.append(tuple(torch.empty_like(q) for _ in range(3)))
        works.append(torch.empty(binding.workspace_bytes(B, N, H, d), dtype=torch.uint8, device=dev))
    for s, cfg, (q, k, v, do), (o, lse), g, ws in zip(streams, CASES, data, fwd, grads, works):
        with torch.cuda.stream(s):
            binding.bwd_into(q, k, v, o, lse, do, *g, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r), ws, stream=s)
    torch.cuda.synchronize()
    fa.check()
    for cfg, (dq_r, dk_r, dv_r), (dq, dk, dv) in zip(CASES, ref, grads):
        assert torch.equal(dk, dk_r), f"{cfg.name}: dK differs"
        assert torch.equal(dv, dv_r), f"{cfg.name}: dV differs"
        ulp = torch.maximum(dq_r.float().abs(), torch.full_like(dq_r.float(), 1e-3)) * 2.0 ** -7
        assert bool(((dq.float() - dq_r.float()).abs() <= 4 * ulp).all()), f"{cfg.name}: dQ differs"
