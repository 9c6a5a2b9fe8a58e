"""Work and byte counts of an attention call (measurement bookkeeping, host only).

FLOPs follow the usual convention of two GEMMs in the forward and five in the
backward over the visible (query, key) pairs: forward = 4·d·pairs,
backward = 10·d·pairs. Pairs are counted exactly under the causal / window mask
("FlashAttention技术解析：加速GPT训练的核心优化" §2.1 gives the O(N²d) per-layer cost;
the mask removes the invisible pairs from it).

Beside the exact count, the tile-granular count charges every 128 x 128 (query tile, key
tile) block that holds at least one visible pair in full, as a tiled kernel that skips only
whole masked tiles would compute it.

Algorithmic HBM bytes: forward reads Q, K, V and writes O (4 bf16 tensors) plus
the fp32 LSE; backward reads Q, K, V, O, dO and LSE and writes dQ, dK, dV.
"""

from __future__ import annotations


def visible_pairs(N: int, causal: bool, win_l: int, win_r: int) -> int:
    """Number of (i, j) with key j visible to query i (inclusive window, -1 unbounded)."""
    wr = 0 if causal else win_r
    total = 0
    # Closed form per row, summed by pieces: row i sees [max(0, i-wl), min(N-1, i+wr)].
    for i in range(N):
        lo = max(0, i - win_l) if win_l >= 0 else 0
        hi = min(N - 1, i + wr) if wr >= 0 else N - 1
        total += max(0, hi - lo + 1)
    return total


def flops(B: int, N: int, H: int, d: int, causal: bool, win_l: int, win_r: int) -> tuple[int, int]:
    """(forward FLOPs, backward FLOPs) over all heads."""
    p = visible_pairs(N, causal, win_l, win_r) * B * H
    return 4 * d * p, 10 * d * p


def visible_tile_pairs(N: int, causal: bool, win_l: int, win_r: int, tile: int = 128) -> int:
    """Number of (query tile, key tile) blocks of `tile` x `tile` holding at least one visible pair."""
    wr = 0 if causal else win_r
    nt = (N + tile - 1) // tile
    total = 0
    for i in range(nt):
        r0, r1 = i * tile, min(N, (i + 1) * tile) - 1
        lo = max(0, r0 - win_l) if win_l >= 0 else 0  # the first row sees furthest left
        hi = min(N - 1, r1 + wr) if wr >= 0 else N - 1  # the last row sees furthest right
        if hi >= lo:
            total += hi // tile - lo // tile + 1
    return total


def flops_tile_granular(B: int, N: int, H: int, d: int, causal: bool, win_l: int, win_r: int,
                        tile: int = 128) -> tuple[int, int]:
    """(forward, backward) FLOPs counting every touched tile x tile block in full."""
    p = visible_tile_pairs(N, causal, win_l, win_r, tile) * tile * tile * B * H
    return 4 * d * p, 10 * d * p


def hbm_bytes(B: int, N: int, H: int, d: int) -> tuple[int, int]:
    """(forward bytes, backward bytes): 4T+L and 8T+L with T one bf16 tensor, L one fp32 row vector."""
    t = B * N * H * d * 2
    l_ = B * H * N * 4
    return 4 * t + l_, 8 * t + l_
