"""E4M3 decoding and the FP8 forward of exact attention, in float64.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The CUDA
library never calls it, and it shares no code with the CUDA path.

What it computes:

* "突破大模型训练瓶颈：Flash-Attention编译优化与内存占用解决方案" (adg.csdn.net),
  section "混合精度计算": attention on FP16, BF16 or FP8 inputs, the FP8 path taking
  ``q_descale`` and ``k_descale`` arguments for the conversion.

Readings taken where the page is silent (also listed with the design notes):

* Q, K and V arrive as E4M3 codes (one byte per element), each with a descale
  factor per (batch, head): the number a code stands for is
  ``descale[b, h] * decode(code)``. The page names only ``q_descale`` and
  ``k_descale``; V is FP8 as well, so it gets a ``v_descale`` of the same form.
* The attention itself is the plain definition (``attention_fp64``) applied to
  those dequantised values; the FP8 step adds nothing else.
* E4M3 follows the OCP 8-bit floating point specification: 1 sign bit, 4 exponent
  bits with bias 7, 3 mantissa bits; exponent field 0 encodes the subnormals
  m/8 * 2^-6; S.1111.111 is NaN; there are no infinities; the largest finite
  value is 448.

Layout: codes are uint8 arrays (B, N, H, d); descales are float arrays (B, H).
"""

from __future__ import annotations

import numpy as np

from oracle import attention_fp64

E4M3_BIAS = 7
E4M3_MAX = 448.0


def decode_e4m3(codes) -> np.ndarray:
    """float64 value of every E4M3 code (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp = (c >> 3) & 0xF
    man = (c & 0x7).astype(np.float64)
    normal = (1.0 + man / 8.0) * np.exp2(exp - E4M3_BIAS)
    subnormal = (man / 8.0) * np.exp2(1 - E4M3_BIAS)
    val = sign * np.where(exp == 0, subnormal, normal)
    return np.where((exp == 0xF) & ((c & 0x7) == 0x7), np.nan, val)


def dequantize(codes, descale) -> np.ndarray:
    """(B, N, H, d) codes and (B, H) descales -> float64 values descale[b, h] * decode(code)."""
    vals = decode_e4m3(codes)
    ds = np.asarray(descale, dtype=np.float64)
    return vals * ds[:, None, :, None]


def attention_forward_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale, causal=False, win_l=-1, win_r=-1,
                          heads=None, block_rows=None):
    """(O, LSE) of attention on dequantised E4M3 inputs; O (B, N, H, d), LSE (B, H, N)."""
    q = dequantize(q8, q_descale)
    k = dequantize(k8, k_descale)
    v = dequantize(v8, v_descale)
    return attention_fp64.attention_forward(q, k, v, scale, causal, win_l, win_r, heads=heads,
                                            block_rows=block_rows)


def forward_rows_fp8(q8, k8, v8, q_descale, k_descale, v_descale, b, h, rows, scale, causal=False, win_l=-1,
                     win_r=-1):
    """O and LSE of the listed query rows of head (b, h) (for sampled checks at full size)."""
    qd = np.asarray(q_descale, dtype=np.float64)[b, h]
    kd = np.asarray(k_descale, dtype=np.float64)[b, h]
    vd = np.asarray(v_descale, dtype=np.float64)[b, h]
    q = decode_e4m3(q8[b, :, h]) * qd
    k = decode_e4m3(k8[b, :, h]) * kd
    v = decode_e4m3(v8[b, :, h]) * vd
    return attention_fp64.forward_rows(q[None, :, None], k[None, :, None], v[None, :, None], 0, 0, rows, scale,
                                       causal, win_l, win_r)
