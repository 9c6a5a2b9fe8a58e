"""The multi-process path on the CPU: two gloo ranks on 127.0.0.1.

Covers the helpers bench.py uses when launched with torch.distributed.run (rank discovery,
process group with a timeout, barrier, max-over-ranks timing, whole-job aggregate) and the
batch sharding: attention computed per rank on its own batch shard (here by the fp64 oracle,
since this runs without a GPU) and gathered equals the unsharded result — the problems are
independent, so no collective is needed on the data path.
"""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from exact_attention_116_b200 import distributed as mg


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist

    from exact_attention_116_b200.inputs import make_custom
    from oracle import attention_fp64 as oracle

    info = mg.rank_info()
    assert (info.world, info.rank) == (world, rank)
    mg.init(info, "gloo", timeout_s=60)
    try:
        mg.barrier(info)
        cpu = torch.device("cpu")
        # timing: the job's time is the slowest rank's
        assert mg.max_over_ranks(info, 1.5 + rank, cpu) == 1.5 + (world - 1)
        assert mg.aggregate_rate(10.0, world, 2.0) == 10.0 * world / 2.0
        # sharded forward over the batch == unsharded forward
        B, N, H, d = 3, 40, 2, 16
        q, k, v, _ = (x.double().numpy() for x in make_custom(B, N, H, d, seed=7))
        b0, b1 = mg.shard_batch(B, world, rank)
        o_local, lse_local = oracle.attention_forward(q[b0:b1], k[b0:b1], v[b0:b1], 0.25, True)
        sizes = [mg.shard_batch(B, world, r) for r in range(world)]
        pad = max(e - s for s, e in sizes)
        o_pad = torch.zeros(pad, N, H, d, dtype=torch.float64)
        o_pad[: b1 - b0] = torch.from_numpy(o_local)
        gathered = [torch.zeros_like(o_pad) for _ in range(world)]
        dist.all_gather(gathered, o_pad)  # result collection only, as a caller would do
        o_all = np.concatenate([g[: e - s].numpy() for g, (s, e) in zip(gathered, sizes)])
        o_ref, _ = oracle.attention_forward(q, k, v, 0.25, True)
        assert np.abs(o_all - o_ref).max() < 1e-12
        mg.barrier(info)
    finally:
        mg.shutdown(info)


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks(world):
    mp.spawn(_worker, args=(world, _free_port()), nprocs=world, join=True)


def test_shard_batch_partitions():
    for B in range(1, 12):
        for world in range(1, 9):
            ranges = [mg.shard_batch(B, world, r) for r in range(world)]
            covered = [b for s, e in ranges for b in range(s, e)]
            assert covered == list(range(B))
            sizes = [e - s for s, e in ranges]
            assert max(sizes) - min(sizes) <= 1
