"""Attention over a batch of variable-length sequences packed along the token axis, in float64.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The CUDA
library never calls it, and it shares no code with the CUDA path.

What it computes ("Flash Attention V2核心网络算子解析" §五, dynamic shapes / variable
sequence lengths): the sequences of a batch have different lengths; they are stored one
after another, sequence b occupying token rows [cu_seqlens[b], cu_seqlens[b+1]) of
(total, H, d) arrays. Each sequence is attended on its own, exactly as the plain
definition (``attention_fp64``) does for a single sequence: positions, causal masking and
windows count from the sequence's first token, and no token sees another sequence.

Readings taken where the pages are silent (also listed with the design notes):

* ``cu_seqlens`` is (B + 1,) int with cu_seqlens[0] = 0, non-decreasing, cu_seqlens[B] =
  total (empty sequences allowed).
* LSE is laid out (H, total): row t of head h is token t of the packed batch.
"""

from __future__ import annotations

import numpy as np

from oracle import attention_fp64


def _check_cu(cu_seqlens, total: int) -> np.ndarray:
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    assert cu.ndim == 1 and cu[0] == 0 and cu[-1] == total and (np.diff(cu) >= 0).all()
    return cu


def varlen_forward(q, k, v, cu_seqlens, scale, causal=False, win_l=-1, win_r=-1, alibi_slopes=None):
    """(O (total, H, d), LSE (H, total)) of packed sequences; alibi_slopes optional (H,)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    total, H, d = q.shape
    cu = _check_cu(cu_seqlens, total)
    o = np.zeros((total, H, d))
    lse = np.full((H, total), -np.inf)
    for b in range(len(cu) - 1):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        if t1 == t0:
            continue
        sl = None if alibi_slopes is None else np.asarray(alibi_slopes, dtype=np.float64)[None, :]
        ob, lb = attention_fp64.attention_forward(q[None, t0:t1], k[None, t0:t1], v[None, t0:t1], scale, causal,
                                                  win_l, win_r, alibi_slopes=sl)
        o[t0:t1] = ob[0]
        lse[:, t0:t1] = lb[0]
    return o, lse


def varlen_backward(q, k, v, do, cu_seqlens, scale, causal=False, win_l=-1, win_r=-1, alibi_slopes=None):
    """(dQ, dK, dV) (total, H, d) of L = sum(dO * O) for packed sequences."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    total = q.shape[0]
    cu = _check_cu(cu_seqlens, total)
    grads = [np.zeros_like(q) for _ in range(3)]
    for b in range(len(cu) - 1):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        if t1 == t0:
            continue
        sl = None if alibi_slopes is None else np.asarray(alibi_slopes, dtype=np.float64)[None, :]
        g = attention_fp64.attention_backward(q[None, t0:t1], k[None, t0:t1], v[None, t0:t1], do[None, t0:t1], scale,
                                              causal, win_l, win_r, alibi_slopes=sl)
        for out, gb in zip(grads, g[:3]):
            out[t0:t1] = gb[0]
    return tuple(grads)
