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


# The E4M3 forward is measured on the training shape.
FP8_CONFIGS: dict[str, AttnConfig] = {
    "train_fwd_fp8": AttnConfig("train_fwd_fp8", 2, 8192, 16, 128, True, seed=106, backward=False,
                                note="B2 H16 N8192 d128 causal, E4M3 Q/K/V with per-head descales, forward only"),
}

E4M3_MAX = 448.0


def make_fp8_inputs(cfg: AttnConfig, *, seed: int | None = None, shape: tuple[int, int, int, int] | None = None):
    """Return host (q8, k8, v8) uint8 E4M3 codes (B, N, H, d) and float32 (q_descale, k_descale, v_descale) (B, H).

    Q, K, V are drawn as in ``make_inputs`` (float32 N(0, 1), same generator and order, times
    ``cfg.qk_mult`` for Q and K); each (b, h) slice gets descale = max|x| / 448 and its codes are
    torch's round-to-nearest-even float8_e4m3fn conversion of x / descale.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed if seed is None else seed)
    shp = cfg.shape if shape is None else shape
    codes, descales = [], []
    for i in range(3):
        x = torch.randn(shp, generator=g, dtype=torch.float32)
        if i < 2 and cfg.qk_mult != 1.0:
            x.mul_(cfg.qk_mult)
        amax = x.abs().amax(dim=(1, 3))                      # (B, H)
        ds = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
        y = (x / ds[:, None, :, None]).clamp_(-E4M3_MAX, E4M3_MAX)
        codes.append(y.to(torch.float8_e4m3fn).view(torch.uint8).contiguous())
        descales.append(ds.contiguous())
    return tuple(codes), tuple(descales)


@dataclass(frozen=True)
class DecodeConfig:
    """A KV-cache decode workload: B sequences of ragged length, Sq new rows each, paged cache."""

    name: str
    B: int
    Sq: int
    H: int
    d: int
    len_lo: int
    len_hi: int
    page_size: int
    causal: bool = True
    win_l: int = -1
    win_r: int = -1
    seed: int = 0
    spare_pages: int = 3
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    @property
    def max_pages(self) -> int:
        return (self.len_hi + self.page_size - 1) // self.page_size


DECODE_CONFIGS: dict[str, DecodeConfig] = {
    "decode_paged": DecodeConfig("decode_paged", 8, 1, 16, 128, 4096, 8192, 256, True, seed=107,
                                 note="B8 H16 d128, 1 new row per sequence, context 4096-8192 keys (uniform), "
                                      "256-key pages in random order"),
    "decode_paged_sq4": DecodeConfig("decode_paged_sq4", 8, 4, 16, 128, 4096, 8192, 256, True, seed=108,
                                     note="B8 H16 d128, 4 new rows per sequence (a speculative step), context "
                                          "4096-8192 keys (uniform), 256-key pages in random order"),
}


def make_decode_inputs(cfg: DecodeConfig, *, seed: int | None = None):
    """Return host tensors (q, k_cache, v_cache, block_table, seqlens).

    Draw order from ``torch.Generator('cpu').manual_seed(seed)``: q (B, Sq, H, d), the K page
    pool, the V page pool (each (B * max_pages + spare, page_size, H, d)), all float32 N(0, 1)
    rounded to bf16; then the lengths, uniform integers in [len_lo, len_hi]; then a random
    permutation of the pages, sequence b taking entries [b * max_pages, (b + 1) * max_pages).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed if seed is None else seed)
    num_pages = cfg.B * cfg.max_pages + cfg.spare_pages
    q = torch.randn((cfg.B, cfg.Sq, cfg.H, cfg.d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    kc = torch.randn((num_pages, cfg.page_size, cfg.H, cfg.d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    vc = torch.randn((num_pages, cfg.page_size, cfg.H, cfg.d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    seqlens = torch.randint(cfg.len_lo, cfg.len_hi + 1, (cfg.B,), generator=g, dtype=torch.int64).to(torch.int32)
    perm = torch.randperm(num_pages, generator=g)[: cfg.B * cfg.max_pages]
    block_table = perm.reshape(cfg.B, cfg.max_pages).to(torch.int32).contiguous()
    return q, kc, vc, block_table, seqlens


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
