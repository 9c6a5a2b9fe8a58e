"""fp64 CPU oracle for exact scaled-dot-product attention, forward and backward.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The CUDA
library never calls it, and it shares no code with the CUDA path.

What it computes is the plain definition, written out with numpy in float64 and
the full score rows materialised before normalisation (no online softmax):

* "Flash Attention V2核心网络算子解析" (yunthe.com), §二.1, the attention formula:
  Attention(Q,K,V) = softmax(Q Kᵀ · scale) V.
* "FlashAttention技术解析：加速GPT训练的核心优化" (pwwt.cn), §2.1: the N×N score
  matrix the standard algorithm stores; §2.2: the call's ``causal``,
  ``window_size=(left, right)`` with -1 meaning unbounded, and
  ``softmax_scale`` defaulting to 1/sqrt(head_dim).
* "突破大模型训练瓶颈：Flash-Attention编译优化与内存占用解决方案" (adg.csdn.net),
  section "滑动窗口注意力": ``window_size=(128, 128)`` as a left/right window.

Readings taken where the pages are silent (each is also listed with the design notes):

* Window bounds are inclusive: key j is visible to query i iff
  0 <= j < N, (win_l == -1 or j >= i - win_l), (win_r' == -1 or j <= i + win_r').
* ``causal`` forces win_r' = 0 (queries and keys have the same length, so the
  diagonal is unambiguous); otherwise win_r' = win_r.
* LSE is the natural-log log-sum-exp of the scaled, masked scores of a row.
* A row with no visible key (impossible for valid windows, because j = i is
  always visible) gets O = 0 and LSE = -inf.
* Backward is the exact derivative of L = sum(dO * O) with respect to Q, K, V;
  there is no upstream gradient into LSE.
* ALiBi (the call's ``alibi_slopes``, "FlashAttention技术解析" §2.2, which passes None for
  "no positional bias"): with a slope m for the head, the score of query i and key j gets
  -m * |i - j| added after scaling, before the mask and the softmax. The slopes are
  constants of the call (no gradient); the backward uses the biased P.

Layout: q, k, v, dO are (B, N, H, d) arrays (any float dtype; they are widened to
float64 exactly). LSE and D are (B, H, N).
"""

from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def effective_right(causal: bool, win_r: int) -> int:
    """Right window bound actually applied: 0 under causal masking, else win_r."""
    return 0 if causal else int(win_r)


def visible_mask(rows: np.ndarray, n_keys: int, causal: bool, win_l: int, win_r: int) -> np.ndarray:
    """Boolean matrix M[r, j] = key j visible to query rows[r] (inclusive window)."""
    wr = effective_right(causal, win_r)
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(n_keys, dtype=np.int64)[None, :]
    vis = np.ones((i.shape[0], n_keys), dtype=bool)
    if win_l >= 0:
        vis &= j >= i - win_l
    if wr >= 0:
        vis &= j <= i + wr
    return vis


def visible_key_span(r0: int, r1: int, n_keys: int, causal: bool, win_l: int, win_r: int) -> tuple[int, int]:
    """Half-open range of keys that any query row in [r0, r1) can see.

    Keys outside the range are masked for every row of the block, so leaving
    them out of a block's score rows changes no sum (each would add exp(-inf)=0).
    """
    wr = effective_right(causal, win_r)
    lo = max(0, r0 - win_l) if win_l >= 0 else 0
    hi = min(n_keys, (r1 - 1) + wr + 1) if wr >= 0 else n_keys
    return lo, max(lo, hi)


def _head_scores(q: np.ndarray, k: np.ndarray, rows: np.ndarray, cols: slice,
                 scale: float, causal: bool, win_l: int, win_r: int, alibi: float = 0.0) -> np.ndarray:
    """Scaled, masked scores S[r, c] = scale * q[rows[r]] . k[c] - alibi * |rows[r] - c| for keys in cols."""
    s = scale * (q[rows] @ k[cols].T)
    if alibi != 0.0:
        keys = np.arange(k.shape[0], dtype=np.int64)[cols]
        s = s - alibi * np.abs(np.asarray(rows, dtype=np.int64)[:, None] - keys[None, :])
    vis = visible_mask(rows, k.shape[0], causal, win_l, win_r)[:, cols]
    return np.where(vis, s, NEG_INF)


def _softmax_rows(s: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Row softmax of a complete score block and its natural-log LSE.

    m = max_j s_j, P_j = exp(s_j - m) / sum_j exp(s_j - m), LSE = m + ln sum_j exp(s_j - m).
    Rows with every entry -inf give P = 0 and LSE = -inf.
    """
    m = s.max(axis=1)
    dead = ~np.isfinite(m)
    m_safe = np.where(dead, 0.0, m)
    e = np.exp(s - m_safe[:, None])
    l = e.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(dead[:, None], 0.0, e / np.where(dead, 1.0, l)[:, None])
        lse = np.where(dead, NEG_INF, m_safe + np.log(np.where(dead, 1.0, l)))
    return p, lse


def _row_blocks(n: int, block_rows: int | None):
    step = n if not block_rows else max(1, int(block_rows))
    for r0 in range(0, n, step):
        yield r0, min(n, r0 + step)


def head_forward(q, k, v, scale, causal=False, win_l=-1, win_r=-1, block_rows=None, alibi=0.0):
    """Forward for one (b, h): q, k, v are (N, d) float64. Returns (O (N,d), LSE (N,)).

    ``block_rows`` only bounds memory: each block holds complete score rows, so
    the softmax of every row is still taken over its full visible key set.
    """
    n = q.shape[0]
    o = np.zeros((n, v.shape[1]), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    for r0, r1 in _row_blocks(n, block_rows):
        c0, c1 = visible_key_span(r0, r1, k.shape[0], causal, win_l, win_r)
        rows = np.arange(r0, r1)
        s = _head_scores(q, k, rows, slice(c0, c1), scale, causal, win_l, win_r, alibi)
        p, lse[r0:r1] = _softmax_rows(s)
        o[r0:r1] = p @ v[c0:c1]
    return o, lse


def head_probs(q, k, scale, causal=False, win_l=-1, win_r=-1, alibi=0.0):
    """Full softmax matrix P (N, N) of one head (small N only; used by the pins)."""
    n = q.shape[0]
    s = _head_scores(q, k, np.arange(n), slice(0, k.shape[0]), scale, causal, win_l, win_r, alibi)
    return _softmax_rows(s)[0]


def head_backward(q, k, v, do, scale, causal=False, win_l=-1, win_r=-1, block_rows=None, alibi=0.0):
    """Gradients of L = sum(dO * O) for one head. Returns (dQ, dK, dV, D).

    With P the softmax matrix of the forward:
      dV = Pᵀ dO;  dP = dO Vᵀ;  D_i = sum_j P_ij dP_ij;  dS = P * (dP - D);
      dQ = scale * dS K;  dK = scale * dSᵀ Q.
    The row blocks recompute P from complete score rows (the same quantity the
    forward normalises), and dK, dV are summed over the blocks.
    """
    n = q.shape[0]
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros_like(k, dtype=np.float64)
    dv = np.zeros_like(v, dtype=np.float64)
    dvec = np.zeros(n, dtype=np.float64)
    for r0, r1 in _row_blocks(n, block_rows):
        backward_rows(q, k, v, do, r0, r1, scale, causal, win_l, win_r, dq, dk, dv, dvec, alibi)
    return dq, dk, dv, dvec


def backward_rows(q, k, v, do, r0, r1, scale, causal, win_l, win_r, dq, dk, dv, dvec, alibi=0.0):
    """Contribution of query rows [r0, r1) of one head to the gradients (added into dk, dv;
    dq and dvec rows [r0, r1) written). Summing it over a partition of the rows gives the
    whole backward."""
    c0, c1 = visible_key_span(r0, r1, k.shape[0], causal, win_l, win_r)
    rows = np.arange(r0, r1)
    s = _head_scores(q, k, rows, slice(c0, c1), scale, causal, win_l, win_r, alibi)
    p, _ = _softmax_rows(s)
    g = do[r0:r1]
    dv[c0:c1] += p.T @ g
    dp = g @ v[c0:c1].T
    d_i = (p * dp).sum(axis=1)
    ds = p * (dp - d_i[:, None])
    dq[r0:r1] = scale * (ds @ k[c0:c1])
    dk[c0:c1] += scale * (ds.T @ q[r0:r1])
    dvec[r0:r1] = d_i


def _as_f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _slope(alibi_slopes, b: int, h: int) -> float:
    return 0.0 if alibi_slopes is None else float(np.asarray(alibi_slopes, dtype=np.float64)[b, h])


def attention_forward(q, k, v, scale, causal=False, win_l=-1, win_r=-1, heads=None, block_rows=None,
                      alibi_slopes=None):
    """Forward over (B, N, H, d) inputs. Returns O (B,N,H,d) and LSE (B,H,N), float64.

    ``heads``: optional list of (b, h) pairs; heads not listed are left as NaN.
    ``alibi_slopes``: optional (B, H) slopes (ALiBi bias -m * |i - j|).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    b_, n, h_, d = q.shape
    o = np.full((b_, n, h_, d), np.nan)
    lse = np.full((b_, h_, n), np.nan)
    for b, h in (heads if heads is not None else [(b, h) for b in range(b_) for h in range(h_)]):
        o[b, :, h, :], lse[b, h, :] = head_forward(q[b, :, h], k[b, :, h], v[b, :, h], scale,
                                                   causal, win_l, win_r, block_rows, _slope(alibi_slopes, b, h))
    return o, lse


def attention_backward(q, k, v, do, scale, causal=False, win_l=-1, win_r=-1, heads=None, block_rows=None,
                       alibi_slopes=None):
    """Backward over (B, N, H, d) inputs. Returns dQ, dK, dV (B,N,H,d) and D (B,H,N), float64."""
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    b_, n, h_, d = q.shape
    dq = np.full((b_, n, h_, d), np.nan)
    dk = np.full_like(dq, np.nan)
    dv = np.full_like(dq, np.nan)
    dvec = np.full((b_, h_, n), np.nan)
    for b, h in (heads if heads is not None else [(b, h) for b in range(b_) for h in range(h_)]):
        g = head_backward(q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], scale,
                          causal, win_l, win_r, block_rows, _slope(alibi_slopes, b, h))
        dq[b, :, h], dk[b, :, h], dv[b, :, h], dvec[b, h] = g
    return dq, dk, dv, dvec


def forward_rows(q, k, v, b, h, rows, scale, causal=False, win_l=-1, win_r=-1, alibi_slopes=None):
    """O and LSE of selected query rows of one head, each computed on its own.

    Used to check sampled outputs at sizes where a whole head is too costly.
    """
    q, k, v = _as_f64(q[b, :, h]), _as_f64(k[b, :, h]), _as_f64(v[b, :, h])
    rows = np.asarray(rows, dtype=np.int64)
    s = _head_scores(q, k, rows, slice(0, k.shape[0]), scale, causal, win_l, win_r, _slope(alibi_slopes, b, h))
    p, lse = _softmax_rows(s)
    return p @ v, lse
