"""Build and call the scalar C oracle (``scalar_attention.c``) — TEST INFRASTRUCTURE."""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "scalar_attention.c")
LIB = os.path.join(_HERE, "_scalar_attention.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc into oracle/_scalar_attention.so."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", "-o", LIB, SRC, "-lm"])
    return LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        i, dbl = ctypes.c_int, ctypes.c_double
        lib.scalar_attention_fwd.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, dbl, i, i, i]
        lib.scalar_attention_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, dbl, i, i, i]
        lib.scalar_attention_fwd.restype = i
        lib.scalar_attention_bwd.restype = i
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def forward(q, k, v, scale, causal=False, win_l=-1, win_r=-1):
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    b, n, h, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((b, h, n))
    rc = _load().scalar_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                      b, n, h, d, float(scale), int(causal), int(win_l), int(win_r))
    if rc != 0:
        raise ValueError("scalar_attention_fwd rejected its arguments")
    return o, lse


def backward(q, k, v, do, scale, causal=False, win_l=-1, win_r=-1):
    q, k, v, do = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, do))
    b, n, h, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = _load().scalar_attention_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                                      b, n, h, d, float(scale), int(causal), int(win_l), int(win_r))
    if rc != 0:
        raise ValueError("scalar_attention_bwd rejected its arguments")
    return dq, dk, dv
