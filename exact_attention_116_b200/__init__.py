"""Exact scaled-dot-product attention for NVIDIA B200 (sm_100a).

The computation lives in a C-ABI CUDA library (``include/fa_sm100.h``, built in-tree as
``libfa_sm100.so``); ``binding`` is its thin ctypes layer. Importing this package loads
nothing: the library is loaded on the first call, which raises if it is missing.
"""

from .binding import (  # noqa: F401
    FaError,
    FlashAttention,
    attention_bwd,
    attention_bwd_varlen,
    attention_decode_paged,
    attention_fwd,
    attention_fwd_fp8,
    attention_fwd_varlen,
    bwd_into,
    bwd_stages,
    check,
    decode_paged_into,
    decode_splits,
    decode_workspace_bytes,
    flash_attention,
    fwd_fp8_into,
    fwd_into,
    load,
    workspace_bytes,
)
