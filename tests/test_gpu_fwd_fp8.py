"""GPU parity of the E4M3 forward (fa_fwd_fp8, through the C ABI) against the fp64 oracle.

The oracle decodes the same codes, applies the same descales and computes the plain
definition. The kernel's only rounding beyond the bf16 path's is P: the unnormalised
probabilities (in (0, 2^8], the lazy-rescale bound) are rounded to E4M3 for P·V, while the
row sums use the unrounded values. Tolerances, from that:

* per row i and column c, |ΔO_ic| <= 2^-4 · max_{j visible} |V_jc| (+ the bf16 output half-ulp):
  E4M3 round-to-nearest has relative error <= 2^-4 in its normal range, so the weights
  w_j = P_j / l move by at most 2^-4 · w_j and sum_j w_j |V_jc| <= max_j |V_jc|. (P below
  E4M3's normal range, 2^-6, has absolute error <= 2^-10 against l >= 1; with zero-mean
  rounding these add up to far less than the bound at the sizes tested.)
* relative RMS error of O over a head <= 2^-4/sqrt(3) ~ 0.036: each weight carries an
  independent relative rounding error whose RMS is at most 2^-4/sqrt(3) (uniform over half an
  E4M3 spacing, which is 2^-4 of the value at the bottom of a binade and 2^-5 at the top).
  The error of a row and the row itself are both averages over the same keys, so their ratio
  does not shrink with the number of keys: the relative RMS of O is of the order of that of
  one weight (measured 0.020-0.024 on N(0,1) inputs).
* max |ΔLSE| <= 1e-3, as for bf16: products of E4M3 values are exact in fp32 and the row
  sum is taken before rounding P.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_116_b200 as fa
from exact_attention_116_b200.inputs import FP8_CONFIGS, AttnConfig, make_fp8_inputs
from oracle import fp8_e4m3 as oracle8

pytestmark = pytest.mark.gpu

ROW_BOUND = 2.0 ** -4
BF16_HALF_ULP = 2.0 ** -9
RMS_TOL = 2.0 ** -4 / np.sqrt(3.0)
LSE_TOL = 1e-3


def run_fp8(codes, descales, scale, causal, win):
    dev = [t.cuda() for t in (*codes, *descales)]
    o, lse = fa.attention_fwd_fp8(*dev, scale, causal, win)
    fa.check()
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def assert_fp8_close(o, lse, o_ref, lse_ref, vmax, what):
    """o, o_ref (..., rows, d); vmax (..., rows, d): max |V_jc| over the keys row i sees."""
    assert np.isfinite(o).all() and np.isfinite(lse).all(), what
    err = np.abs(o - o_ref)
    bound = ROW_BOUND * vmax + BF16_HALF_ULP * np.maximum(1.0, np.abs(o_ref))
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{what}: O error {worst:.2f} x the E4M3 bound"
    rms = float(np.sqrt((err ** 2).mean()) / max(np.sqrt((o_ref ** 2).mean()), 1e-30))
    assert rms <= RMS_TOL, f"{what}: relative RMS error {rms:.3e}"
    e_lse = float(np.abs(lse - lse_ref).max())
    assert e_lse <= LSE_TOL, f"{what}: LSE error {e_lse:.3e}"
    return worst, rms, e_lse


def visible_vmax(v, rows, causal, wl, wr):
    """max_j |v_j| (per column) over the keys each listed row sees; v (N, d) float64."""
    n = v.shape[0]
    out = np.empty((len(rows), v.shape[1]))
    wr_eff = 0 if causal else wr
    for r, i in enumerate(rows):
        lo = max(0, i - wl) if wl >= 0 else 0
        hi = min(n - 1, i + wr_eff) if wr_eff >= 0 else n - 1
        out[r] = np.abs(v[lo:hi + 1]).max(axis=0)
    return out


def check_whole(B, N, H, causal, win, seed, scale=None, qk_mult=1.0):
    cfg = AttnConfig("custom_fp8", B, N, H, 128, causal, win[0], win[1], seed=seed, qk_mult=qk_mult)
    codes, descales = make_fp8_inputs(cfg)
    sc = 1.0 / np.sqrt(128) if scale is None else scale
    o, lse = run_fp8(codes, descales, sc, causal, win)
    cn = [t.numpy() for t in codes]
    dn = [t.numpy().astype(np.float64) for t in descales]
    o_ref, lse_ref = oracle8.attention_forward_fp8(*cn, *dn, sc, causal, *win)
    v = oracle8.dequantize(cn[2], dn[2])
    for b in range(B):
        for h in range(H):
            vmax = visible_vmax(v[b, :, h], range(N), causal, *win)
            assert_fp8_close(o[b, :, h], lse[b, h], o_ref[b, :, h], lse_ref[b, h], vmax,
                             f"B{B} N{N} H{H} causal={causal} win={win} head {(b, h)}")


EDGE_CASES = [
    (1, 1, 1, False, (-1, -1)),
    (1, 127, 2, True, (-1, -1)),
    (2, 129, 1, False, (-1, -1)),
    (1, 300, 2, False, (5, 3)),
    (1, 513, 1, False, (0, 0)),
    (1, 384, 2, True, (100, -1)),
    (1, 700, 2, False, (128, 128)),
    (2, 1000, 3, True, (-1, -1)),
]


@pytest.mark.parametrize("B,N,H,causal,win", EDGE_CASES)
def test_fp8_fwd_edge_shapes(B, N, H, causal, win):
    check_whole(B, N, H, causal, win, seed=4000 + N + H)


@pytest.mark.parametrize("scale", [-0.1, 0.0, 0.25])
def test_fp8_fwd_scale_values(scale):
    check_whole(1, 260, 2, True, (-1, -1), seed=41, scale=scale)


def test_fp8_fwd_large_logits_and_many_items():
    """Q and K x8 before quantisation (descales x8); 3 x 24 heads: several items per CTA."""
    check_whole(3, 600, 24, False, (-1, -1), seed=42, qk_mult=8.0)


def test_fp8_fwd_per_head_descales_are_applied_per_head():
    cfg = AttnConfig("custom_fp8", 1, 256, 2, 128, False, seed=43)
    (q8, k8, v8), (qd, kd, vd) = make_fp8_inputs(cfg)
    o1, l1 = run_fp8((q8, k8, v8), (qd, kd, vd), 0.1, False, (-1, -1))
    # doubling head 1's v_descale doubles its O and leaves head 0 and every LSE untouched
    vd2 = vd.clone()
    vd2[0, 1] *= 2
    o2, l2 = run_fp8((q8, k8, v8), (qd, kd, vd2), 0.1, False, (-1, -1))
    assert np.array_equal(o2[:, :, 0], o1[:, :, 0]) and np.array_equal(l1, l2)
    assert np.allclose(o2[:, :, 1], 2 * o1[:, :, 1], rtol=2 ** -8, atol=0)


def test_fp8_fwd_train_shape_sampled_rows():
    cfg = FP8_CONFIGS["train_fwd_fp8"]
    codes, descales = make_fp8_inputs(cfg)
    o, lse = run_fp8(codes, descales, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r))
    o2, lse2 = run_fp8(codes, descales, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r))
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2), "FP8 forward is not bitwise reproducible"
    cn = [t.numpy() for t in codes]
    dn = [t.numpy().astype(np.float64) for t in descales]
    rng = np.random.default_rng(7)
    rows = sorted(set([0, 1, 127, 128, 255, 256, cfg.N // 2, cfg.N - 129, cfg.N - 1] +
                      rng.integers(0, cfg.N, 30).tolist()))
    for b, h in [(0, 0), (cfg.B - 1, cfg.H - 1), (1, 5)]:
        o_ref, lse_ref = oracle8.forward_rows_fp8(*cn, *dn, b, h, rows, cfg.scale, cfg.causal, cfg.win_l, cfg.win_r)
        v = oracle8.decode_e4m3(cn[2][b, :, h]) * dn[2][b, h]
        vmax = visible_vmax(v, rows, cfg.causal, cfg.win_l, cfg.win_r)
        assert_fp8_close(o[b, rows, h], lse[b, h, rows], o_ref, lse_ref, vmax, f"train_fwd_fp8 head {(b, h)}")
