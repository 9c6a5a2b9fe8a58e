"""Seeded synthetic inputs for exact attention — shared by the tests, the bench and the oracle checks.

This module draws numbers and nothing else: it holds none of attention's arithmetic.

Recipe (the pages measure on no dataset; their workloads are GPT-style shapes):
``torch.Generator('cpu').manual_seed(seed)``, then ``torch.randn`` in float32 for
Q, K, V, dO in that order, each of shape (B, N, H, d); a config may multiply Q and K
by a power of two (exact in bf16) to produce large logits; finally round to bf16
(round-to-nearest-even). The same host tensors feed the GPU and the oracle.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class AttnConfig:
    """One workload: shapes, mask and seed."""

    name: str
    B: int
    N: int
    H: int
    d: int
    causal: bool
    win_l: int = -1
    win_r: int = -1
    seed: int = 0
    qk_mult: float = 1.0
    backward: bool = True
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    @property
    def shape(self) -> tuple[int, int, int, int]:
        return (self.B, self.N, self.H, self.d)


# The five workloads the build is measured and checked on.
CONFIGS: dict[str, AttnConfig] = {
    "tiny_fwd": AttnConfig("tiny_fwd", 1, 128, 2, 64, False, seed=101, backward=False,
                           note="B1 H2 N128 d64 non-causal, forward only"),
    "gpt_fwd": AttnConfig("gpt_fwd", 4, 2048, 16, 64, True, seed=102, backward=False,
                          note="B4 H16 N2048 d64 causal, forward only"),
    "train_fwd_bwd": AttnConfig("train_fwd_bwd", 2, 8192, 16, 128, True, seed=103,
                                note="B2 H16 N8192 d128 causal, forward + backward"),
    "long_fwd_bwd": AttnConfig("long_fwd_bwd", 1, 32768, 16, 128, True, seed=104,
                               note="B1 H16 N32768 d128 causal, forward + backward"),
    "window_fwd_bwd": AttnConfig("window_fwd_bwd", 2, 16384, 16, 64, False, 128, 128, seed=105, qk_mult=8.0,
                                 note="B2 H16 N16384 d64 window (128,128), Q and K x8, forward + backward"),
}


def make_inputs(cfg: AttnConfig, *, seed: int | None = None, shape: tuple[int, int, int, int] | None = None,
                qk_mult: float | None = None):
    """Return host bf16 tensors (q, k, v, do), each (B, N, H, d), drawn in that order."""
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed if seed is None else seed)
    shp = cfg.shape if shape is None else shape
    mult = cfg.qk_mult if qk_mult is None else qk_mult
    out = []
    for i in range(4):
        x = torch.randn(shp, generator=g, dtype=torch.float32)
        if i < 2 and mult != 1.0:
            x.mul_(mult)
        out.append(x.to(torch.bfloat16))
    return tuple(out)


def make_custom(B: int, N: int, H: int, d: int, seed: int, qk_mult: float = 1.0):
    """Inputs of an arbitrary shape with the same recipe (edge-case tests)."""
    cfg = AttnConfig("custom", B, N, H, d, False, seed=seed, qk_mult=qk_mult)
    return make_inputs(cfg)
