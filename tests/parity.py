"""Shared helpers of the GPU parity tests: run the CUDA path and compare with the oracle.

Tolerances (bf16 inputs and outputs, fp32 accumulation):
* forward: every element obeys |O_gpu - O_ref| <= 1e-2 + ulp_bf16(O_gpu) / 2, and
  max |LSE_gpu - LSE_ref| <= 1e-3. The kernel rounds its fp32 result o32 to bf16 once at the end,
  so |O_gpu - O_ref| <= |O_gpu - o32| + |o32 - O_ref| <= ulp/2 + |o32 - O_ref|: the check is
  exactly the 1e-2 bound on the kernel's own error plus that last rounding, which alone can
  exceed 1e-2 (bf16's half-ulp in [4, 8) is 2^-6 ~ 0.0156). The raw maximum is reported too.
* backward: relative L2 error ||g - g_ref|| / ||g_ref|| <= 1e-2 per gradient (per sampled head
  at the large sizes). Where the exact dQ or dK vanishes (a query that sees only itself has
  dS = 0 exactly, so dQ = dK = 0), the GPU returns rounding noise of (dP - D) and the
  quotient is meaningless; the denominator is then floored at 1e-3 * ||dV_ref||, the scale
  of the gradients that cannot vanish (sum_j dV_j = sum_i dO_i).
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import attention_fp64 as oracle

FWD_O_TOL = 1e-2
FWD_LSE_TOL = 1e-3
BWD_REL_L2_TOL = 1e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def window_args(causal: bool, win: tuple[int, int]):
    return bool(causal), int(win[0]), int(win[1])


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 values at |x| (8 significant bits): 2^(e - 8) for |x| in [2^e, 2^(e+1))."""
    _, e = np.frexp(np.abs(np.asarray(x, dtype=np.float64)))  # |x| = m 2^e with m in [0.5, 1)
    return np.ldexp(1.0, e - 9)


def fwd_errors(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray):
    """(O error beyond the output's last rounding, raw max O error, max LSE error) over the refs' rows."""
    diff = np.abs(o_gpu - o_ref)
    excess = diff - half_ulp_bf16(o_gpu)
    return float(excess.max()), float(diff.max()), float(np.abs(lse_gpu - lse_ref).max())


def assert_fwd_close(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    e_o, e_raw, e_lse = fwd_errors(o_gpu, lse_gpu, o_ref, lse_ref)
    assert np.isfinite(o_gpu).all() and np.isfinite(lse_gpu).all(), what
    assert e_o <= FWD_O_TOL, f"{what}: O error {e_o:.3e} beyond the bf16 output rounding (raw {e_raw:.3e})"
    assert e_lse <= FWD_LSE_TOL, f"{what}: LSE error {e_lse:.3e}"
    return e_o, e_raw, e_lse


def rel_l2(g: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30))


def assert_bwd_close(grads_gpu, grads_ref, what=""):
    errs = []
    floor = 1e-3 * float(np.linalg.norm(grads_ref[2]))
    for name, g, r in zip(("dQ", "dK", "dV"), grads_gpu, grads_ref):
        assert np.isfinite(g).all(), f"{what}: {name} not finite"
        e = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), floor, 1e-30))
        errs.append(e)
        assert e <= BWD_REL_L2_TOL, f"{what}: {name} relative L2 error {e:.3e}"
    return errs
