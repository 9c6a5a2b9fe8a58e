"""Blocked online-softmax recomputation of the attention forward, in float64.

TEST INFRASTRUCTURE (see ``attention_fp64``): it exists only to pin the direct
oracle. It restates the tiled algorithm the pages describe, independently of the
direct definition, so that the two can be compared:

* "FlashAttention技术解析：加速GPT训练的核心优化", §1 item 3: each block keeps
  running statistics (the maximum and the sum) and renormalises.
* "FlashAttention 剖析", §3: scores of one block, a local softmax, accumulation of
  the weighted V blocks, and normalisation across blocks.
* "Flash Attention V2核心网络算子解析", §二.1 step 2: the incremental log-domain
  update of the running log-sum-exp. The printed snippet has lost the sum over
  the new block's scores; the reading used here is
  lse' = m + ln( sum_j exp(s_j - m) + exp(lse - m) ),  m = max(lse, max_j s_j).

Keys are visited in blocks in any order the caller gives; the result must not
depend on that order (up to rounding).
"""

from __future__ import annotations

import numpy as np

from .attention_fp64 import visible_mask  # the mask rule only; no softmax code is shared

NEG_INF = -np.inf


def lse_merge(lse: np.ndarray, s_block: np.ndarray) -> np.ndarray:
    """Running natural-log LSE after folding in one block of scores (rows x keys)."""
    m = np.maximum(lse, s_block.max(axis=1))
    dead = ~np.isfinite(m)
    m0 = np.where(dead, 0.0, m)
    tot = np.exp(s_block - m0[:, None]).sum(axis=1) + np.exp(lse - m0)
    with np.errstate(divide="ignore"):
        return np.where(dead, NEG_INF, m0 + np.log(tot))


def head_forward_online(q, k, v, scale, causal=False, win_l=-1, win_r=-1, block=16, order=None):
    """Forward of one head by key blocks with running (max, sum, accumulator).

    Returns (O, LSE_from_stats, LSE_from_merge): the LSE both from the running
    max/sum and from chained ``lse_merge`` calls.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    n, nk = q.shape[0], k.shape[0]
    blocks = [(c, min(nk, c + block)) for c in range(0, nk, block)]
    if order is not None:
        blocks = [blocks[i] for i in order]
    rows = np.arange(n)
    vis = visible_mask(rows, nk, causal, win_l, win_r)
    m = np.full(n, NEG_INF)
    l = np.zeros(n)
    acc = np.zeros((n, v.shape[1]))
    lse_chain = np.full(n, NEG_INF)
    for c0, c1 in blocks:
        s = np.where(vis[:, c0:c1], scale * (q @ k[c0:c1].T), NEG_INF)
        lse_chain = lse_merge(lse_chain, s)
        m_new = np.maximum(m, s.max(axis=1))
        live = np.isfinite(m_new)
        ref = np.where(live, m_new, 0.0)
        alpha = np.where(np.isfinite(m), np.exp(m - ref), 0.0)
        p = np.exp(s - ref[:, None])
        l = alpha * l + p.sum(axis=1)
        acc = alpha[:, None] * acc + p @ v[c0:c1]
        m = m_new
    with np.errstate(divide="ignore", invalid="ignore"):
        o = np.where(l[:, None] > 0, acc / np.where(l > 0, l, 1.0)[:, None], 0.0)
        lse = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), NEG_INF)
    return o, lse, lse_chain
