"""fp64 CPU oracle for exact attention — TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package. The CUDA library never routes through it.

* ``attention_fp64``       — the definition, numpy float64 (the oracle proper).
* ``online_softmax_fp64``  — a blocked online-softmax restatement (a pin only).
* ``scalar_attention.c``   — scalar C loops (a second implementation; a pin only).
* ``scalar_ref``           — builds and loads the C pin through ctypes.
"""

from .attention_fp64 import (  # noqa: F401
    attention_backward,
    attention_forward,
    forward_rows,
    head_backward,
    head_forward,
    head_probs,
    visible_key_span,
    visible_mask,
)
