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
    assert bench.recorded_traffic("no_such_kernel") is None
    h1 = bench.kernel_source_hash(["fa_fwd.cuh", "sm100_ptx.cuh"])
    assert h1 == bench.kernel_source_hash(["fa_fwd.cuh", "sm100_ptx.cuh"]) and len(h1) == 16
    assert h1 != bench.kernel_source_hash(["fa_bwd.cuh", "sm100_ptx.cuh"])
