"""Multi-GPU plumbing for data-parallel attention (host side only).

Every (batch, head) problem is independent in the forward and the backward, so the work
shards across GPUs with no collective on the data path. This module holds the little that
multi-process runs need: rank discovery from the torch.distributed.run environment, process
group set-up with a short timeout, a barrier, the max-over-ranks reduction used for timing,
the whole-job aggregate, and an even split of the batch dimension. The backend is a
parameter ("nccl" on GPUs, "gloo" on the CPU) so the same code runs in CPU tests.
"""

from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankInfo:
    world: int
    rank: int
    local_rank: int

    @property
    def is_root(self) -> bool:
        return self.rank == 0


def rank_info() -> RankInfo:
    """World size, rank and local rank from the launcher's environment (1, 0, 0 when absent)."""
    return RankInfo(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(info: RankInfo, backend: str, timeout_s: float = 120.0, device: torch.device | None = None) -> None:
    """Join the process group (no-op for a single process)."""
    if info.world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if backend == "nccl" and device is not None else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def shutdown(info: RankInfo) -> None:
    if info.world > 1 and dist.is_initialized():
        dist.destroy_process_group()


def barrier(info: RankInfo) -> None:
    if info.world > 1:
        dist.barrier()


def max_over_ranks(info: RankInfo, x: float, device: torch.device) -> float:
    """The largest value of x over all ranks (timing is the slowest rank's)."""
    if info.world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds


def shard_batch(B: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous batch range [b0, b1) of this rank; ranks' ranges partition [0, B)."""
    base, extra = divmod(B, world)
    b0 = rank * base + min(rank, extra)
    return b0, b0 + base + (1 if rank < extra else 0)
