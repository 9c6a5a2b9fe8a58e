"""ctypes binding of the fa_sm100 C ABI (include/fa_sm100.h): argument marshalling only.

Every step of the computation runs in the CUDA library. There is no CPU or PyTorch
fallback: if the library is missing or the tensors are not on a CUDA device, the calls
raise.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa_sm100.so")

FA_OK = 0
STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_CUDA",
                4: "FA_ERR_TIMEOUT", 5: "FA_ERR_NO_MEMORY", 6: "FA_ERR_DEVICE"}
EXPORTS = ("fa_fwd", "fa_fwd_ex", "fa_fwd_varlen", "fa_fwd_fp8", "fa_decode_splits", "fa_decode_workspace_bytes", "fa_decode_paged",
           "fa_bwd_workspace_bytes", "fa_bwd", "fa_bwd_ex", "fa_bwd_varlen", "fa_bwd_deterministic", "fa_bwd_preprocess",
           "fa_bwd_main", "fa_bwd_dq_convert", "fa_bwd_static_workspace", "fa_check", "fa_status_string")

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load() -> ctypes.CDLL:
    """Load the in-tree CUDA library (built by ``exact_attention_116_b200.build``)."""
    global _lib
    if _lib is None:
        _lib = open_library(LIB_PATH)
    return _lib


def open_library(path: str) -> ctypes.CDLL:
    """Open a build of the C ABI (the library or its bounds-checking variant, libfa_sm100_debug.so)
    and declare its argument types. Every wrapper here calls the one ``load()`` returns."""
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
    lib.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
    lib.fa_fwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
    lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
    lib.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, i, vp, sz, vp]
    lib.fa_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, i, vp, sz, vp]
    lib.fa_decode_splits.argtypes = [i, i, i, i, i]
    lib.fa_decode_splits.restype = i
    lib.fa_decode_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.fa_decode_workspace_bytes.restype = sz
    lib.fa_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i, i, vp, sz,
                                    vp]
    lib.fa_bwd_workspace_bytes.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_bytes.restype = sz
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp, sz, vp]
    lib.fa_bwd_deterministic.argtypes = lib.fa_bwd.argtypes
    lib.fa_bwd_preprocess.argtypes = [vp, vp, vp, i, i, i, i, vp, sz, vp]
    lib.fa_bwd_main.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp, sz, vp]
    lib.fa_bwd_dq_convert.argtypes = [vp, i, i, i, i, vp, sz, vp]
    lib.fa_check.argtypes = [vp]
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_bwd_static_workspace.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
    for name in ("fa_fwd", "fa_fwd_ex", "fa_bwd_ex", "fa_fwd_varlen", "fa_bwd_varlen", "fa_fwd_fp8", "fa_decode_paged",
                 "fa_bwd", "fa_bwd_deterministic", "fa_bwd_preprocess", "fa_bwd_main", "fa_bwd_dq_convert",
                 "fa_bwd_static_workspace", "fa_check"):
        getattr(lib, name).restype = i
    return lib


def status_string(status: int) -> str:
    try:
        return load().fa_status_string(int(status)).decode()
    except RuntimeError:
        return STATUS_NAMES.get(int(status), "FA_ERR_UNKNOWN")


def _raise(status: int, where: str) -> None:
    if status != FA_OK:
        raise FaError(status, where)


def _stream_handle(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check_qkv(*ts: torch.Tensor, dtype=torch.bfloat16) -> tuple[int, int, int, int]:
    shape = ts[0].shape
    if len(shape) != 4:
        raise ValueError("tensors must be (batch, seq, heads, head_dim)")
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (there is no CPU path)")
        if t.dtype != dtype:
            raise ValueError(f"tensors must be {dtype}")
        if t.shape != shape or not t.is_contiguous():
            raise ValueError("tensors must be contiguous and of equal shape")
    return tuple(int(x) for x in shape)  # type: ignore[return-value]


def _check_lse(lse: torch.Tensor, shape: tuple[int, ...]) -> None:
    """LSE / row statistics: a contiguous float32 CUDA tensor of the given shape. Checked before any
    launch: the C layer sees only a pointer, so a wrong dtype or layout would be read out of bounds."""
    if lse.dtype != torch.float32:
        raise ValueError(f"lse must be float32 (got {lse.dtype})")
    if tuple(lse.shape) != tuple(shape):
        raise ValueError(f"lse must have shape {tuple(shape)} (got {tuple(lse.shape)})")
    if not lse.is_contiguous():
        raise ValueError("lse must be contiguous")
    if not lse.is_cuda:
        raise ValueError("lse must be on a CUDA device (there is no CPU path)")


def _check_workspace(workspace) -> tuple[int | None, int]:
    """Optional backward workspace: a contiguous uint8 CUDA tensor; returns (pointer, bytes)."""
    if workspace is None:
        return None, 0
    if workspace.dtype != torch.uint8:
        raise ValueError(f"workspace must be a uint8 tensor (got {workspace.dtype})")
    if not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    if not workspace.is_cuda:
        raise ValueError("workspace must be on a CUDA device")
    return workspace.data_ptr(), workspace.numel()


def _scale(scale: float | None, d: int) -> float:
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def _check_slopes(alibi_slopes, B: int, H: int):
    if alibi_slopes is None:
        return None
    t = alibi_slopes
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, H):
        raise ValueError("alibi_slopes must be a contiguous (B, H) float32 CUDA tensor")
    return t.data_ptr()


def fwd_into(q, k, v, o, lse, scale=None, causal=False, window=(-1, -1), stream=None, alibi_slopes=None) -> None:
    """fa_fwd (fa_fwd_ex with ALiBi slopes) into caller-provided o (B,N,H,d) bf16 and lse (B,H,N) fp32."""
    B, N, H, d = _check_qkv(q, k, v, o)
    _check_lse(lse, (B, H, N))
    slopes = _check_slopes(alibi_slopes, B, H)
    if slopes is None:
        st = load().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, N, H, d,
                           _scale(scale, d), int(bool(causal)), int(window[0]), int(window[1]),
                           _stream_handle(stream))
        _raise(st, "fa_fwd")
    else:
        st = load().fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), slopes, o.data_ptr(), lse.data_ptr(), B, N,
                              H, d, _scale(scale, d), int(bool(causal)), int(window[0]), int(window[1]),
                              _stream_handle(stream))
        _raise(st, "fa_fwd_ex")


def attention_fwd(q, k, v, scale=None, causal=False, window=(-1, -1), stream=None, alibi_slopes=None):
    """Forward: returns (o, lse) with o (B,N,H,d) bf16 and lse (B,H,N) fp32 (natural log).
    ``alibi_slopes``: optional (B, H) float32 CUDA tensor (bias -m |i - j|)."""
    B, N, H, d = _check_qkv(q, k, v)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    fwd_into(q, k, v, o, lse, scale, causal, window, stream, alibi_slopes)
    return o, lse


def _as_codes(t: torch.Tensor) -> torch.Tensor:
    """E4M3 tensors may come as torch.float8_e4m3fn or as their uint8 codes."""
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t


def fwd_fp8_into(q8, k8, v8, q_descale, k_descale, v_descale, o, lse, scale=None, causal=False, window=(-1, -1),
                 stream=None) -> None:
    """fa_fwd_fp8: q8, k8, v8 (B,N,H,d) E4M3 codes (uint8 or float8_e4m3fn), descales (B,H) float32,
    into o (B,N,H,d) bf16 and lse (B,H,N) float32."""
    q8, k8, v8 = (_as_codes(t) for t in (q8, k8, v8))
    B, N, H, d = _check_qkv(q8, k8, v8, dtype=torch.uint8)
    _check_qkv(o)
    if tuple(o.shape) != (B, N, H, d):
        raise ValueError("o must have the shape of q")
    _check_lse(lse, (B, H, N))
    for t in (q_descale, k_descale, v_descale):
        if t.dtype != torch.float32 or tuple(t.shape) != (B, H) or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("descales must be contiguous (B, H) float32 CUDA tensors")
    st = load().fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), q_descale.data_ptr(), k_descale.data_ptr(),
                           v_descale.data_ptr(), o.data_ptr(), lse.data_ptr(), B, N, H, d, _scale(scale, d),
                           int(bool(causal)), int(window[0]), int(window[1]), _stream_handle(stream))
    _raise(st, "fa_fwd_fp8")


def attention_fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale=None, causal=False, window=(-1, -1),
                      stream=None):
    """FP8 forward: returns (o, lse), o (B,N,H,d) bf16 and lse (B,H,N) float32."""
    B, N, H, d = q8.shape
    o = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=q8.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    fwd_fp8_into(q8, k8, v8, q_descale, k_descale, v_descale, o, lse, scale, causal, window, stream)
    return o, lse


def workspace_bytes(B: int, N: int, H: int, d: int) -> int:
    return int(load().fa_bwd_workspace_bytes(B, N, H, d))


def bwd_into(q, k, v, o, lse, do, dq, dk, dv, scale=None, causal=False, window=(-1, -1), workspace=None,
             stream=None, deterministic=False, alibi_slopes=None) -> None:
    """fa_bwd (or fa_bwd_deterministic; fa_bwd_ex with ALiBi slopes) into caller-provided dq, dk, dv.
    ``workspace``: uint8 CUDA tensor or None."""
    B, N, H, d = _check_qkv(q, k, v, o, do, dq, dk, dv)
    _check_lse(lse, (B, H, N))
    ws_ptr, ws_bytes = _check_workspace(workspace)
    slopes = _check_slopes(alibi_slopes, B, H)
    lib = load()
    if slopes is not None:
        st = lib.fa_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                           slopes, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, N, H, d, _scale(scale, d),
                           int(bool(causal)), int(window[0]), int(window[1]), int(bool(deterministic)), ws_ptr,
                           ws_bytes, _stream_handle(stream))
        _raise(st, "fa_bwd_ex")
        return
    fn, name = (lib.fa_bwd_deterministic, "fa_bwd_deterministic") if deterministic else (lib.fa_bwd, "fa_bwd")
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr(), B, N, H, d, _scale(scale, d), int(bool(causal)), int(window[0]),
            int(window[1]), ws_ptr, ws_bytes, _stream_handle(stream))
    _raise(st, name)


def attention_bwd(q, k, v, o, lse, do, scale=None, causal=False, window=(-1, -1), workspace=None, stream=None,
                  deterministic=False, alibi_slopes=None):
    """Backward: returns (dq, dk, dv), the gradients of sum(do * o). With deterministic=True the
    result is bitwise reproducible (dQ accumulated per query tile in a fixed order)."""
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    bwd_into(q, k, v, o, lse, do, dq, dk, dv, scale, causal, window, workspace, stream, deterministic, alibi_slopes)
    return dq, dk, dv


def bwd_stages(q, k, v, o, lse, do, dq, dk, dv, workspace, scale=None, causal=False, window=(-1, -1),
               stream=None, between=None) -> None:
    """The three launches of the backward issued one by one; ``between(i)`` runs before stage i
    (i = 0, 1, 2) and once more after the last (i = 3) — e.g. to record CUDA events."""
    B, N, H, d = _check_qkv(q, k, v, o, do, dq, dk, dv)
    _check_lse(lse, (B, H, N))
    if workspace is None:
        raise ValueError("bwd_stages needs a workspace of workspace_bytes(B, N, H, d) bytes")
    ws, wb = _check_workspace(workspace)
    lib, s = load(), _stream_handle(stream)
    sc = _scale(scale, d)
    if between:
        between(0)
    _raise(lib.fa_bwd_preprocess(o.data_ptr(), lse.data_ptr(), do.data_ptr(), B, N, H, d, ws, wb, s),
           "fa_bwd_preprocess")
    if between:
        between(1)
    _raise(lib.fa_bwd_main(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                           B, N, H, d, sc, int(bool(causal)), int(window[0]), int(window[1]), ws, wb, s),
           "fa_bwd_main")
    if between:
        between(2)
    _raise(lib.fa_bwd_dq_convert(dq.data_ptr(), B, N, H, d, ws, wb, s), "fa_bwd_dq_convert")
    if between:
        between(3)


def bwd_into_static_workspace(q, k, v, o, lse, do, dq, dk, dv, scale=None, causal=False, window=(-1, -1),
                              stream=None) -> None:
    """fa_bwd_static_workspace: the backward without any device allocation.

    For callers that may not allocate device memory (an allocator they do not own, a fixed
    memory budget): the scratch is a 32 MiB array inside the library. Larger problems raise
    FaError(FA_ERR_UNSUPPORTED). Calls that overlap on the GPU share that array and race;
    issue them one after another. Make the first call on each device outside stream capture.
    """
    B, N, H, d = _check_qkv(q, k, v, o, do, dq, dk, dv)
    _check_lse(lse, (B, H, N))
    st = load().fa_bwd_static_workspace(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, N, H, d, _scale(scale, d), int(bool(causal)),
            int(window[0]), int(window[1]), _stream_handle(stream))
    _raise(st, "fa_bwd_static_workspace")


def check(stream=None) -> None:
    """Synchronise and raise if a kernel recorded a device-side error (e.g. a wait timeout)."""
    _raise(load().fa_check(_stream_handle(stream)), "fa_check")


class FlashAttention(torch.autograd.Function):
    """autograd wrapper: forward saves (q, k, v, o, lse); backward recomputes the scores."""

    @staticmethod
    def forward(ctx, q, k, v, scale=None, causal=False, window=(-1, -1)):
        o, lse = attention_fwd(q, k, v, scale, causal, window)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.args = (scale, causal, window)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = attention_bwd(q, k, v, o, lse, do.contiguous(), *ctx.args)
        return dq, dk, dv, None, None, None


def flash_attention(q, k, v, scale=None, causal=False, window=(-1, -1)):
    """Differentiable exact attention on (batch, seq, heads, head_dim) bf16 CUDA tensors."""
    return FlashAttention.apply(q, k, v, scale, causal, window)


def decode_paged_into(q, k_cache, v_cache, block_table, seqlens, o, lse, scale=None, causal=False, window=(-1, -1),
                      splits=0, workspace=None, stream=None, k_new=None, v_new=None) -> None:
    """fa_decode_paged: q (B,Sq,H,d) bf16 new rows; k_cache, v_cache (num_pages,page_size,H,d) bf16;
    block_table (B,max_pages) int32; seqlens (B,) int32; into o (B,Sq,H,d) bf16, lse (B,H,Sq) float32.
    k_new, v_new: optional (B,Sq,H,d) bf16 rows written into the caches first (in place).
    splits: CTAs per head (each head's visible tiles, listed sequence after sequence, cut into that
    many equal pieces); 0 = decode_splits(). workspace: decode_workspace_bytes(B,Sq,H,d,splits)
    bytes (any contents), or None to allocate on the stream."""
    B, Sq, H, d = _check_qkv(q, o)
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    if k_new is not None:
        _check_qkv(q, k_new, v_new)
    _check_qkv(k_cache, v_cache)
    num_pages, page_size, Hc, dc = k_cache.shape
    if (Hc, dc) != (H, d):
        raise ValueError("cache heads / head dim must match q")
    for t, name in ((block_table, "block_table"), (seqlens, "seqlens")):
        if t.dtype != torch.int32 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(seqlens.shape) != (B,):
        raise ValueError("block_table must be (B, max_pages) and seqlens (B,)")
    _check_lse(lse, (B, H, Sq))
    ws_ptr, ws_bytes = _check_workspace(workspace)
    kn, vn = (None, None) if k_new is None else (k_new.data_ptr(), v_new.data_ptr())
    st = load().fa_decode_paged(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), kn, vn, block_table.data_ptr(),
                                seqlens.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Sq, H, d, num_pages, page_size,
                                int(block_table.shape[1]), _scale(scale, d), int(bool(causal)), int(window[0]),
                                int(window[1]), int(splits), ws_ptr, ws_bytes, _stream_handle(stream))
    _raise(st, "fa_decode_paged")


def decode_splits(B: int, Sq: int, H: int, d: int, max_keys: int) -> int:
    """The pieces per head fa_decode_paged picks for splits=0 on the current device."""
    n = int(load().fa_decode_splits(B, Sq, H, d, max_keys))
    if n < 0:
        _raise(-n, "fa_decode_splits")
    return n


def decode_workspace_bytes(B: int, Sq: int, H: int, d: int, splits: int) -> int:
    return int(load().fa_decode_workspace_bytes(B, Sq, H, d, splits))


def attention_decode_paged(q, k_cache, v_cache, block_table, seqlens, scale=None, causal=False, window=(-1, -1),
                           splits=0, stream=None, k_new=None, v_new=None):
    """Paged-KV decode: returns (o, lse), o (B,Sq,H,d) bf16 and lse (B,H,Sq) float32. With k_new, v_new the
    new rows are first written into the caches (in place) at positions seqlens[b] - Sq + i."""
    B, Sq, H, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    decode_paged_into(q, k_cache, v_cache, block_table, seqlens, o, lse, scale, causal, window, splits, None, stream,
                      k_new, v_new)
    return o, lse


def _check_packed(cu_seqlens, *ts):
    total, H, d = ts[0].shape
    for t in ts:
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != (total, H, d):
            raise ValueError("packed tensors must be contiguous (total, H, d) bfloat16 CUDA tensors")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1 or \
            not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous (B + 1,) int32 CUDA tensor")
    return int(cu_seqlens.numel()) - 1, total, H, d


def _check_head_slopes(alibi_slopes, H):
    if alibi_slopes is None:
        return None
    if alibi_slopes.dtype != torch.float32 or not alibi_slopes.is_cuda or tuple(alibi_slopes.shape) != (H,) or \
            not alibi_slopes.is_contiguous():
        raise ValueError("alibi_slopes must be a contiguous (H,) float32 CUDA tensor for packed batches")
    return alibi_slopes.data_ptr()


def attention_fwd_varlen(q, k, v, cu_seqlens, scale=None, causal=False, window=(-1, -1), stream=None,
                         alibi_slopes=None):
    """Packed variable-length forward: q, k, v (total, H, d) bf16, cu_seqlens (B + 1,) int32.
    Returns (o (total, H, d) bf16, lse (H, total) float32)."""
    B, total, H, d = _check_packed(cu_seqlens, q, k, v)
    o = torch.empty_like(q)
    lse = torch.empty((H, total), dtype=torch.float32, device=q.device)
    st = load().fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens.data_ptr(),
                              _check_head_slopes(alibi_slopes, H), o.data_ptr(), lse.data_ptr(), B, total, H, d,
                              _scale(scale, d), int(bool(causal)), int(window[0]), int(window[1]),
                              _stream_handle(stream))
    _raise(st, "fa_fwd_varlen")
    return o, lse


def attention_bwd_varlen(q, k, v, o, lse, do, cu_seqlens, scale=None, causal=False, window=(-1, -1), workspace=None,
                         stream=None, deterministic=False, alibi_slopes=None):
    """Backward of attention_fwd_varlen: returns (dq, dk, dv), each (total, H, d) bf16."""
    B, total, H, d = _check_packed(cu_seqlens, q, k, v, o, do)
    _check_lse(lse, (H, total))
    ws_ptr, ws_bytes = _check_workspace(workspace)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = load().fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                              cu_seqlens.data_ptr(), _check_head_slopes(alibi_slopes, H), dq.data_ptr(),
                              dk.data_ptr(), dv.data_ptr(), B, total, H, d, _scale(scale, d), int(bool(causal)),
                              int(window[0]), int(window[1]), int(bool(deterministic)), ws_ptr, ws_bytes,
                              _stream_handle(stream))
    _raise(st, "fa_bwd_varlen")
    return dq, dk, dv
