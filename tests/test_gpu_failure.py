"""Failure detection on the GPU without a fault: a bounded wait runs out.

With FA_DEBUG_DROP_S_SIGNAL=1 the forward kernel's MMA warp withholds one "scores ready"
signal, so a softmax warp waits on an mbarrier that nothing completes. Every wait in the
kernels is bounded (about 2 s); the kernel must give up, record the timeout, and exit, so
that fa_check reports FA_ERR_TIMEOUT and the CUDA context stays usable for the next call.
"""

from __future__ import annotations

import os
import time

import numpy as np
import pytest

import exact_attention_116_b200 as fa
from exact_attention_116_b200.binding import FaError
from exact_attention_116_b200.inputs import make_custom
from oracle import attention_fp64 as oracle

pytestmark = pytest.mark.gpu


def test_withheld_signal_times_out_and_context_survives():
    q, k, v, _ = (x.cuda() for x in make_custom(1, 256, 1, 64, seed=21))
    os.environ["FA_DEBUG_DROP_S_SIGNAL"] = "1"
    try:
        t0 = time.time()
        fa.attention_fwd(q, k, v, None, True)
        with pytest.raises(FaError) as info:
            fa.check()
        assert info.value.status == 4  # FA_ERR_TIMEOUT
        assert time.time() - t0 < 60
    finally:
        del os.environ["FA_DEBUG_DROP_S_SIGNAL"]
    # the error record is cleared and the next call runs normally
    o, lse = fa.attention_fwd(q, k, v, None, True)
    fa.check()
    o_ref, lse_ref = oracle.attention_forward(q.double().cpu().numpy(), k.double().cpu().numpy(),
                                              v.double().cpu().numpy(), 1 / 8, True)
    assert np.abs(o.double().cpu().numpy() - o_ref).max() < 1e-2
    assert np.abs(lse.double().cpu().numpy() - lse_ref).max() < 1e-3
