"""Compile the CUDA library (sm_100a) in-tree: exact_attention_116_b200/libfa_sm100.so.

Run as ``python -m exact_attention_116_b200.build`` or through ``__graft_entry__.build()``.
The library is one translation unit (csrc/fa_api.cu includes the kernels) linked against
the static CUDA runtime; the driver's tensor-map encoder is fetched at run time.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "fa_api.cu")
HEADERS = [os.path.join(PKG, "csrc", f) for f in ("fa_fwd.cuh", "fa_bwd.cuh", "fa_bwd_dq.cuh", "fa_decode.cuh", "sm100_ptx.cuh")] + [
    os.path.join(ROOT, "include", "fa_sm100.h")
]
LIB = os.path.join(PKG, "libfa_sm100.so")
# The same library with device-side bounds checks (-DFA_DEBUG=1): every computed TMA coordinate,
# bulk-copy range, shared-memory destination and global index is checked before use; a failed
# check is reported through fa_check as FA_ERR_DEVICE instead of touching memory out of range.
LIB_DEBUG = os.path.join(PKG, "libfa_sm100_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def command(out: str = LIB, verbose_ptxas: bool = False, extra: list[str] | None = None) -> list[str]:
    cmd = [nvcc_path(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc"), "-o", out, SRC]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    return cmd + list(extra or [])


def needs_build(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(f) > t for f in [SRC, *HEADERS])


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    """Compile the library (or, with debug=True, its bounds-checking variant) if a source changed."""
    out = LIB_DEBUG if debug else LIB
    if force or needs_build(out):
        tmp = out + ".tmp"
        subprocess.check_call(command(tmp, verbose_ptxas, ["-DFA_DEBUG=1"] if debug else None))
        os.replace(tmp, out)
    return out


if __name__ == "__main__":
    dbg = "--debug" in sys.argv
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv, debug=dbg))
