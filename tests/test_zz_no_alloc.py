"""The allocation-free backward (fa_bwd_static_workspace) against the regular fa_bwd.

Some callers cannot allocate device memory (they run under an allocator they do not own,
or inside a fixed memory budget), so the library offers one backward entry point whose
scratch is a fixed 32 MiB array compiled into the library. This file checks, through the
C ABI, that two calls in a row (different shapes, so the shared scratch is reused) give the
same gradients as fa_bwd with a caller-provided workspace, that the calls change no device
memory usage and leave the stream-ordered pool's high-water marks at zero (a control shows
that those marks do record the allocation fa_bwd makes without a workspace), and that a
problem needing more scratch than the array holds is refused.
It is collected last so that, if it fails, every other test has already run.
"""

from __future__ import annotations

import ctypes

import pytest
import torch

import exact_attention_116_b200 as fa
from exact_attention_116_b200 import binding
from exact_attention_116_b200.inputs import make_custom

pytestmark = pytest.mark.gpu

CASES = [  # B, N, H, d, causal, window — both need well under 32 MiB of scratch
    (1, 1500, 4, 128, True, (-1, -1)),
    (2, 700, 3, 64, False, (64, 32)),
]


def _inputs(B, N, H, d, causal, win, seed):
    q, k, v, do = (x.cuda() for x in make_custom(B, N, H, d, seed=seed))
    o, lse = fa.attention_fwd(q, k, v, None, causal, win)
    return q, k, v, o, lse, do


# Stream-ordered allocations (cudaMallocAsync) come from the device's default memory pool and
# may be returned to it by the time the stream is synchronised, so free memory alone cannot
# show that none was made. The pool's high-water marks can: reset them, make the calls, read
# them back (driver API; attribute values from cuda.h's CUmemPool_attribute).
_RESERVED_MEM_HIGH, _USED_MEM_HIGH = 6, 8


def _pool_high_water():
    cu = ctypes.CDLL("libcuda.so.1")
    dev, pool = ctypes.c_int(), ctypes.c_void_p()
    assert cu.cuCtxGetDevice(ctypes.byref(dev)) == 0
    assert cu.cuDeviceGetDefaultMemPool(ctypes.byref(pool), dev) == 0

    def read():
        out = []
        for attr in (_USED_MEM_HIGH, _RESERVED_MEM_HIGH):
            v = ctypes.c_uint64()
            assert cu.cuMemPoolGetAttribute(pool, attr, ctypes.byref(v)) == 0
            out.append(v.value)
        return tuple(out)

    def reset():
        zero = ctypes.c_uint64(0)
        for attr in (_USED_MEM_HIGH, _RESERVED_MEM_HIGH):
            assert cu.cuMemPoolSetAttribute(pool, attr, ctypes.byref(zero)) == 0

    return reset, read


def test_pool_high_water_sees_a_stream_ordered_allocation():
    """Control for the check below: fa_bwd without a workspace allocates on the stream, and the
    default pool's used-memory high-water mark records it."""
    B, N, H, d, causal, win = CASES[0]
    q, k, v, o, lse, do = _inputs(B, N, H, d, causal, win, seed=299)
    torch.cuda.synchronize()
    reset, read = _pool_high_water()
    reset()
    base = read()  # the marks right after the reset (the pool may still hold memory)
    fa.attention_bwd(q, k, v, o, lse, do, None, causal, win, workspace=None)
    fa.check()
    assert read()[0] >= base[0] + fa.workspace_bytes(B, N, H, d)


def test_static_workspace_matches_fa_bwd_on_two_calls_in_a_row():
    refs, runs = [], []
    for i, (B, N, H, d, causal, win) in enumerate(CASES):
        q, k, v, o, lse, do = _inputs(B, N, H, d, causal, win, seed=300 + i)
        ws = torch.empty(fa.workspace_bytes(B, N, H, d), dtype=torch.uint8, device="cuda")
        refs.append(fa.attention_bwd(q, k, v, o, lse, do, None, causal, win, workspace=ws))
        runs.append((q, k, v, o, lse, do, causal, win))
    fa.check()

    outs = [tuple(torch.empty_like(x) for x in (r[0], r[1], r[2])) for r in runs]
    torch.cuda.synchronize()
    reset, read = _pool_high_water()
    reset()
    base = read()
    free_before = torch.cuda.mem_get_info()[0]
    for (q, k, v, o, lse, do, causal, win), (dq, dk, dv) in zip(runs, outs):
        binding.bwd_into_static_workspace(q, k, v, o, lse, do, dq, dk, dv, None, causal, win)
    fa.check()
    assert torch.cuda.mem_get_info()[0] == free_before, "the allocation-free backward changed device memory usage"
    assert read() == base, f"the allocation-free backward allocated from the stream-ordered pool: {read()} vs {base}"

    for (dq_ref, dk_ref, dv_ref), (dq, dk, dv) in zip(refs, outs):
        assert torch.equal(dk, dk_ref) and torch.equal(dv, dv_ref)
        rel = float((dq.float() - dq_ref.float()).norm() / dq_ref.float().norm())
        assert rel < 1e-3, f"dQ differs from fa_bwd by {rel:.2e} (relative L2)"


def test_static_workspace_refuses_problems_larger_than_its_scratch():
    lib = binding.load()
    fn = lib.fa_bwd_static_workspace
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
    fn.restype = i
    base, step = 0x7F0000000000, 1 << 33  # fake, aligned, disjoint: validation fails before any use
    B, N, H, d = 1, 32768, 16, 128
    assert fa.workspace_bytes(B, N, H, d) > 32 << 20
    ptrs = [base + j * step for j in range(9)]
    st = fn(*ptrs, B, N, H, d, 0.088, 1, -1, -1, None)
    assert st == 2, binding.status_string(st)  # FA_ERR_UNSUPPORTED
