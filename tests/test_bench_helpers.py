"""Host-side checks of bench.py's helpers (no GPU): the packed host/device buffers the
end-to-end legs copy in one piece, the decode byte count, and the traffic-record lookup."""

from __future__ import annotations

import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from exact_attention_116_b200.inputs import DECODE_CONFIGS  # noqa: E402


def test_packed_buffers_views_share_one_aligned_buffer():
    specs = [((3, 1, 5, 7), torch.bfloat16), ((3, 9), torch.int32), ((3,), torch.int32), ((2, 5, 1), torch.float32)]
    buf, views = bench.packed_buffers("cpu", specs)
    assert buf.dtype == torch.uint8 and buf.dim() == 1
    end = 0
    for (shape, dt), v in zip(specs, views):
        assert tuple(v.shape) == shape and v.dtype == dt and v.is_contiguous()
        off = v.data_ptr() - buf.data_ptr()
        assert off % 256 == 0 and off >= end  # aligned, in order, not overlapping the previous view
        end = off + v.numel() * v.element_size()
    assert end <= buf.numel()
    for i, v in enumerate(views):  # writes through a view land in the one buffer
        v.fill_(i + 1)
    for i, v in enumerate(views):
        assert bool((v == i + 1).all())


def test_decode_cache_bytes_counts_visible_rows_and_small_tensors():
    cfg = DECODE_CONFIGS["decode_paged"]
    lens = torch.tensor([5, 0, 300], dtype=torch.int32)
    kv = (5 + 0 + 300) * cfg.H * cfg.d * 2 * 2
    small = 2 * cfg.B * cfg.Sq * cfg.H * cfg.d * 2 + cfg.B * cfg.H * cfg.Sq * 4
    assert bench.decode_cache_bytes(cfg, lens) == kv + small


def test_traffic_lookup():
    assert bench.recorded_traffic("no_such_kernel", "train_fwd_bwd") is None
    h1 = bench.kernel_source_hash(["fa_fwd.cuh", "sm100_ptx.cuh"])
    assert h1 == bench.kernel_source_hash(["fa_fwd.cuh", "sm100_ptx.cuh"]) and len(h1) == 16
    assert h1 != bench.kernel_source_hash(["fa_bwd.cuh", "sm100_ptx.cuh"])


def test_tile_granular_count_matches_brute_force_and_the_configs():
    from exact_attention_116_b200.workload import flops, flops_tile_granular, visible_pairs, visible_tile_pairs
    import numpy as np
    for N, causal, wl, wr in [(300, False, -1, -1), (300, True, -1, -1), (700, False, 128, 128), (513, False, 0, 0),
                              (1030, True, 100, -1), (640, False, -1, 200), (1, False, -1, -1)]:
        i = np.arange(N)[:, None]
        j = np.arange(N)[None, :]
        vis = np.ones((N, N), bool)
        if wl >= 0:
            vis &= j >= i - wl
        r = 0 if causal else wr
        if r >= 0:
            vis &= j <= i + r
        nt = (N + 127) // 128
        blocks = sum(bool(vis[a * 128:(a + 1) * 128, b * 128:(b + 1) * 128].any()) for a in range(nt) for b in range(nt))
        assert visible_tile_pairs(N, causal, wl, wr) == blocks
        assert visible_pairs(N, causal, wl, wr) == int(vis.sum())
    # the workloads' forward GFLOP, exact and tile-granular
    assert round(flops(2, 8192, 16, 128, True, -1, -1)[0] / 1e9, 1) == 549.8
    assert round(flops_tile_granular(2, 8192, 16, 128, True, -1, -1)[0] / 1e9, 1) == 558.3
    # 256 key tiles, causal: 256 * 257 / 2 = 32896 blocks per head, each 4 * 128 * 128 * 128 FLOPs
    assert flops_tile_granular(1, 32768, 16, 128, True, -1, -1)[0] == 32896 * 16 * 4 * 128 * 128 * 128
    assert round(flops_tile_granular(4, 2048, 16, 64, True, -1, -1)[0] / 1e9, 2) == 36.51
    assert round(flops_tile_granular(2, 16384, 16, 64, False, 128, 128)[0] / 1e9, 2) == 51.27
