"""Host-side checks of the C ABI: the library loads, exports every symbol include/fa_sm100.h
declares, and rejects invalid arguments before launching anything. No GPU is touched:
every call here fails validation (fake pointers are never dereferenced).
"""

from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

from exact_attention_116_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_sm100.h")

OK, INVALID, UNSUPPORTED = 0, 1, 2
P = 0x7F0000000000  # a 16-byte aligned fake device address, far from anything real
T = 1 << 30         # spacing that keeps fake tensors disjoint


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(fa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_check", "fa_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(binding.EXPORTS)


def test_debug_library_exports_every_declared_symbol():
    """The bounds-checking build (-DFA_DEBUG=1) offers the same C ABI."""
    dbg = binding.open_library(build.build(debug=True))
    for name in declared_functions():
        assert hasattr(dbg, name), name
    assert dbg.fa_status_string(0).decode() == "FA_OK"


def test_status_strings(lib):
    for code, name in binding.STATUS_NAMES.items():
        assert lib.fa_status_string(code).decode().startswith(name)
    assert lib.fa_status_string(99).decode() == "FA_ERR_UNKNOWN"


def test_workspace_bytes(lib):
    def expect(B, N, H, d):
        a = lambda x: (x + 255) // 256 * 256  # noqa: E731
        npad = (N + 127) // 128 * 128
        return a(B * N * H * d * 4) + 2 * a(B * H * npad * 4) + 256  # + the work counter

    for shape in [(1, 1, 1, 64), (2, 8192, 16, 128), (1, 129, 3, 64), (4, 2048, 16, 64)]:
        assert lib.fa_bwd_workspace_bytes(*shape) == expect(*shape)
    assert lib.fa_bwd_workspace_bytes(0, 128, 1, 64) == 0
    assert lib.fa_bwd_workspace_bytes(1, 128, 1, 96) == 0


def _fwd(lib, q=P, k=P + T, v=P + 2 * T, o=P + 3 * T, lse=P + 4 * T, B=1, N=128, H=2, d=64, scale=0.125,
         causal=0, wl=-1, wr=-1):
    return lib.fa_fwd(q, k, v, o, lse, B, N, H, d, ctypes.c_float(scale), causal, wl, wr, None)


@pytest.mark.parametrize("kw,expected", [
    (dict(q=0), INVALID), (dict(k=0), INVALID), (dict(v=0), INVALID), (dict(o=0), INVALID), (dict(lse=0), INVALID),
    (dict(B=0), INVALID), (dict(N=0), INVALID), (dict(H=0), INVALID), (dict(N=-5), INVALID),
    (dict(d=96), UNSUPPORTED), (dict(d=256), UNSUPPORTED), (dict(d=0), INVALID),
    (dict(wl=-2), INVALID), (dict(wr=-7), INVALID),
    (dict(scale=float("nan")), INVALID), (dict(scale=float("inf")), INVALID),
    (dict(q=P + 8), INVALID), (dict(o=P + 3 * T + 2), INVALID), (dict(lse=P + 4 * T + 2), INVALID),
    (dict(o=P), INVALID),            # output aliases q
    (dict(lse=P + T + 64), INVALID),  # lse inside k
])
def test_fwd_rejects_invalid_arguments(lib, kw, expected):
    assert _fwd(lib, **kw) == expected


def _fwd8(lib, q=P, k=P + T, v=P + 2 * T, qd=P + 3 * T, kd=P + 3 * T + 4096, vd=P + 3 * T + 8192, o=P + 4 * T,
          lse=P + 5 * T, B=1, N=128, H=2, d=128, scale=0.1):
    return lib.fa_fwd_fp8(q, k, v, qd, kd, vd, o, lse, B, N, H, d, ctypes.c_float(scale), 0, -1, -1, None)


@pytest.mark.parametrize("kw,expected", [
    (dict(d=64), UNSUPPORTED), (dict(d=96), UNSUPPORTED), (dict(qd=0), INVALID), (dict(vd=0), INVALID),
    (dict(q=P + 8), INVALID), (dict(kd=P + 3 * T + 4098), INVALID), (dict(o=P + 4 * T + 4), INVALID),
    (dict(o=P + 2 * T), INVALID),        # output aliases v
    (dict(lse=P + 3 * T), INVALID),      # lse overlaps q_descale
    (dict(scale=float("nan")), INVALID), (dict(N=0), INVALID),
])
def test_fwd_fp8_rejects_invalid_arguments(lib, kw, expected):
    assert _fwd8(lib, **kw) == expected


def _bwd(lib, ws=P + 9 * T, ws_bytes=None, dq=P + 6 * T, dk=P + 7 * T, dv=P + 8 * T, B=1, N=128, H=2, d=64,
         scale=0.125, wl=-1, wr=-1, fn="fa_bwd"):
    if ws_bytes is None:
        ws_bytes = lib.fa_bwd_workspace_bytes(B, N, H, d) if B > 0 and N > 0 and H > 0 else 0
    return getattr(lib, fn)(P, P + T, P + 2 * T, P + 3 * T, P + 4 * T, P + 5 * T, dq, dk, dv, B, N, H, d,
                            ctypes.c_float(scale), 0, wl, wr, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,expected", [
    (dict(dq=0), INVALID), (dict(B=0), INVALID), (dict(d=80), UNSUPPORTED), (dict(wl=-3), INVALID),
    (dict(scale=float("-inf")), INVALID), (dict(dq=P + 6 * T + 4), INVALID),
    (dict(dk=P), INVALID),                      # dk aliases q
    (dict(dv=P + 6 * T + 1024), INVALID),       # dv overlaps dq
    (dict(ws=P + 9 * T + 16), INVALID),         # workspace not 256-byte aligned
    (dict(ws_bytes=1024), INVALID),             # workspace too small
    (dict(ws=P + 5 * T), INVALID),              # workspace overlaps dO
])
@pytest.mark.parametrize("fn", ["fa_bwd", "fa_bwd_deterministic"])
def test_bwd_rejects_invalid_arguments(lib, kw, expected, fn):
    assert _bwd(lib, fn=fn, **kw) == expected


def test_bwd_stage_calls_reject_invalid_arguments(lib):
    wsb = lib.fa_bwd_workspace_bytes(1, 128, 2, 64)
    assert lib.fa_bwd_preprocess(P, P + T, P + 2 * T, 1, 128, 2, 64, 0, wsb, None) == INVALID
    assert lib.fa_bwd_main(P, P + T, P + 2 * T, P + 3 * T, P + 4 * T, P + 5 * T, 1, 128, 2, 64,
                           ctypes.c_float(0.1), 0, -1, -1, P + 6 * T, 16, None) == INVALID
    assert lib.fa_bwd_dq_convert(P + 8, 1, 128, 2, 64, P + 6 * T, wsb, None) == INVALID
    assert lib.fa_bwd_dq_convert(P, 1, 128, 2, 48, P + 6 * T, wsb, None) == UNSUPPORTED


def test_decode_workspace_bytes(lib):
    def expect(B, Sq, H, d, pieces):
        a = lambda x: (x + 255) // 256 * 256  # noqa: E731
        rows = (B + pieces - 1) * H * Sq  # (sequence, piece) slots
        return a(rows * d * 4) + a(rows * 4) + a(B * H * 4)  # partial O, partial LSE, arrival counters

    for shape in [(3, 2, 4, 128, 6), (8, 1, 16, 128, 8), (1, 8, 1, 64, 2), (5, 3, 7, 64, 40)]:
        assert lib.fa_decode_workspace_bytes(*shape) == expect(*shape)
    assert lib.fa_decode_workspace_bytes(8, 1, 16, 128, 1) == 0  # one split: nothing to merge
    assert lib.fa_decode_workspace_bytes(8, 1, 16, 96, 4) == 0
    assert lib.fa_decode_workspace_bytes(0, 1, 16, 128, 4) == 0


def _decode(lib, q=P, kc=P + T, vc=P + 2 * T, kn=None, vn=None, table=P + 3 * T, lens=P + 4 * T, o=P + 5 * T,
            lse=P + 6 * T, B=2, Sq=1, H=2, d=128, num_pages=4, page_size=64, max_pages=2, scale=0.1, splits=0,
            ws=None, ws_bytes=0):
    return lib.fa_decode_paged(q, kc, vc, kn, vn, table, lens, o, lse, B, Sq, H, d, num_pages, page_size, max_pages,
                               ctypes.c_float(scale), 1, -1, -1, splits, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,expected", [
    (dict(q=0), INVALID), (dict(table=0), INVALID), (dict(B=0), INVALID), (dict(Sq=0), INVALID),
    (dict(Sq=9), UNSUPPORTED), (dict(d=96), UNSUPPORTED), (dict(page_size=96), UNSUPPORTED),
    (dict(splits=-1), INVALID), (dict(splits=70000), INVALID),
    (dict(kn=P + 7 * T), INVALID),                    # k_new without v_new
    (dict(o=P + 8), INVALID), (dict(lse=P + 6 * T + 2), INVALID),
    (dict(o=P), INVALID),                             # output aliases q
    (dict(vc=P + T + 1024), INVALID),                 # the caches overlap
    (dict(kn=P + 7 * T, vn=P + 8 * T, table=P + T + 64), INVALID),  # a written cache overlaps the table
    (dict(scale=float("nan")), INVALID),
])
def test_decode_rejects_invalid_arguments(lib, kw, expected):
    assert _decode(lib, **kw) == expected


def test_decode_splits_rejects_invalid_arguments(lib):
    assert lib.fa_decode_splits(0, 1, 16, 128, 4096) == -INVALID
    assert lib.fa_decode_splits(8, 0, 16, 128, 4096) == -INVALID
    assert lib.fa_decode_splits(8, 1, 16, 128, 0) == -INVALID
    assert lib.fa_decode_splits(8, 9, 16, 128, 4096) == -UNSUPPORTED
    assert lib.fa_decode_splits(8, 1, 16, 96, 4096) == -UNSUPPORTED


def test_binding_has_no_cpu_path():
    q = torch.zeros(1, 16, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.attention_fwd(q, q, q)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="not built"):
        binding.load()


def _no_launch(*_a, **_k):
    raise AssertionError("validation passed: the call would have reached the library")


def _qkv_any_device(*ts, dtype=torch.bfloat16):
    """_check_qkv without its CUDA requirement, so that the later checks run on CPU tensors."""
    shape = ts[0].shape
    for t in ts:
        assert t.dtype == dtype and t.shape == shape
    return tuple(int(x) for x in shape)


@pytest.mark.parametrize("case", ["dtype", "shape", "transposed", "cpu"])
def test_backward_wrappers_validate_lse_before_any_launch(monkeypatch, case):
    """A bf16, mis-shaped, non-contiguous or host LSE is refused by every backward wrapper
    before the library is touched (the C layer only checks its pointer's alignment)."""
    monkeypatch.setattr(binding, "_check_qkv", _qkv_any_device)
    monkeypatch.setattr(binding, "load", _no_launch)
    B, N, H, d = 1, 16, 2, 64
    t = torch.zeros(B, N, H, d, dtype=torch.bfloat16)
    lse = {"dtype": torch.zeros(B, H, N, dtype=torch.bfloat16),
           "shape": torch.zeros(B, N, H, dtype=torch.float32),
           "transposed": torch.zeros(B, N, H, dtype=torch.float32).transpose(1, 2),
           "cpu": torch.zeros(B, H, N, dtype=torch.float32)}[case]
    msg = {"dtype": "float32", "shape": "shape", "transposed": "contiguous", "cpu": "CUDA"}[case]
    ws = torch.zeros(64, dtype=torch.uint8)
    calls = [
        lambda: binding.bwd_into(t, t, t, t, lse, t, t, t, t),
        lambda: binding.bwd_stages(t, t, t, t, lse, t, t, t, t, ws),
        lambda: binding.bwd_into_static_workspace(t, t, t, t, lse, t, t, t, t),
        lambda: binding.fwd_into(t, t, t, t, lse),
    ]
    for call in calls:
        with pytest.raises(ValueError, match=msg):
            call()


@pytest.mark.parametrize("case", ["dtype", "strided", "cpu"])
def test_backward_wrappers_validate_workspace_before_any_launch(monkeypatch, case):
    monkeypatch.setattr(binding, "_check_qkv", _qkv_any_device)
    monkeypatch.setattr(binding, "_check_lse", lambda *_a: None)
    monkeypatch.setattr(binding, "load", _no_launch)
    t = torch.zeros(1, 16, 2, 64, dtype=torch.bfloat16)
    ws = {"dtype": torch.zeros(64, dtype=torch.float32),
          "strided": torch.zeros(128, dtype=torch.uint8)[::2],
          "cpu": torch.zeros(64, dtype=torch.uint8)}[case]
    msg = {"dtype": "uint8", "strided": "contiguous", "cpu": "CUDA"}[case]
    for call in (lambda: binding.bwd_into(t, t, t, t, None, t, t, t, t, workspace=ws),
                 lambda: binding.bwd_stages(t, t, t, t, None, t, t, t, t, ws)):
        with pytest.raises(ValueError, match=msg):
            call()
    with pytest.raises(ValueError, match="workspace"):
        binding.bwd_stages(t, t, t, t, None, t, t, t, t, None)
