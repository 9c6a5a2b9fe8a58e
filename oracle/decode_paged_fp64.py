"""Attention of new query rows against a paged KV cache (decoding), in float64.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The CUDA
library never calls it, and it shares no code with the CUDA path.

What it computes:

* "FlashAttention技术解析：加速GPT训练的核心优化" (pwwt.cn), §5: FlashDecoding, attention
  over the KV cache at inference time.
* "突破大模型训练瓶颈：Flash-Attention编译优化与内存占用解决方案" (adg.csdn.net), sections
  "Paged KV Cache支持" and the closing list ("启用Paged KV Cache：flash_attn_with_kvcache"):
  the KV cache is held in fixed-size pages that need not be contiguous, and a block table
  (``block_table``) lists the pages of every sequence.

Readings taken where the pages are silent (also listed with the design notes):

* The cache is two arrays (num_pages, page_size, H, d); ``block_table`` is (B, max_pages)
  int32 and ``seqlens`` (B,) int32 is the number of keys sequence b holds. Key j of
  sequence b (0 <= j < seqlens[b]) is row ``j % page_size`` of page
  ``block_table[b, j // page_size]``; entries past the last used page are not read.
* The Sq query rows of a sequence are its newest tokens, already written to the cache:
  query row i sits at position ``pos = seqlens[b] - Sq + i``.
* Masks are those of the training path, taken at ``pos``: causal keeps keys j <= pos; a
  (left, right) window keeps pos - left <= j <= pos + right (inclusive, -1 unbounded).
* New rows' keys and values, when given (``k_new``, ``v_new``: (B, Sq, H, d)), are written
  into the cache at those positions first, as ``flash_attn_with_kvcache`` updates its cache
  in place; rows whose position is negative (a sequence shorter than Sq) are not placed.
* Otherwise the plain definition: O = softmax(scale * q . k) V over the visible keys, and
  LSE the natural-log log-sum-exp of the scaled scores (a row without keys: O = 0,
  LSE = -inf).

Layout: q and O (B, Sq, H, d); LSE (B, H, Sq).
"""

from __future__ import annotations

import numpy as np

from oracle import attention_fp64


def gather_sequence(cache, block_table, b: int, seqlen: int, page_size: int) -> np.ndarray:
    """The (seqlen, H, d) keys (or values) of sequence b, page by page in block-table order."""
    cache = np.asarray(cache)
    rows = []
    for j in range(seqlen):
        rows.append(cache[int(block_table[b, j // page_size]), j % page_size])
    return np.asarray(rows, dtype=np.float64).reshape(seqlen, *cache.shape[2:])


def append_rows(cache, rows, block_table, seqlens, page_size):
    """A copy of the cache with rows[b, i] placed at position seqlens[b] - Sq + i of sequence b."""
    out = np.array(cache, dtype=np.float64, copy=True)
    rows = np.asarray(rows, dtype=np.float64)
    Sq = rows.shape[1]
    for b in range(rows.shape[0]):
        for i in range(Sq):
            pos = int(seqlens[b]) - Sq + i
            if pos >= 0:
                out[int(block_table[b, pos // page_size]), pos % page_size] = rows[b, i]
    return out


def decode_forward(q, k_cache, v_cache, block_table, seqlens, scale, causal=False, win_l=-1, win_r=-1, k_new=None,
                   v_new=None):
    """(O, LSE) of the new query rows of every sequence against its cached keys and values."""
    q = np.asarray(q, dtype=np.float64)
    B, Sq, H, d = q.shape
    page_size = np.asarray(k_cache).shape[1]
    if k_new is not None:
        k_cache = append_rows(k_cache, k_new, block_table, seqlens, page_size)
        v_cache = append_rows(v_cache, v_new, block_table, seqlens, page_size)
    o = np.zeros((B, Sq, H, d))
    lse = np.full((B, H, Sq), -np.inf)
    for b in range(B):
        n = int(seqlens[b])
        if n == 0:  # no keys: every row keeps O = 0, LSE = -inf
            continue
        k = gather_sequence(k_cache, block_table, b, n, page_size)
        v = gather_sequence(v_cache, block_table, b, n, page_size)
        pos = np.arange(n - Sq, n, dtype=np.int64)
        vis = attention_fp64.visible_mask(pos, n, causal, win_l, win_r)
        for h in range(H):
            s = np.where(vis, scale * (q[b, :, h] @ k[:, h].T), -np.inf)
            p, lse[b, h] = attention_fp64._softmax_rows(s)
            o[b, :, h] = p @ v[:, h]
    return o, lse
