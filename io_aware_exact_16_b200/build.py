"""Builds the CUDA library ``libfa.so`` in-tree for sm_100a with nvcc, and its checking twin
``libfa_debug.so`` (the same sources compiled with FA_DEBUG: every plain global load and store
in the kernels checks its index against the buffer it belongs to, records FA_ERR_INVALID_ARG
and skips the access when it is out of range; nothing traps).

The library is the C ABI of ``include/fa.h``; the Python binding in this package loads it
with ctypes.  Run ``python io_aware_exact_16_b200/build.py`` (a plain script: importing the
package first would try to load the library it builds).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libfa.so")
SO_DEBUG = os.path.join(HERE, "libfa_debug.so")
SOURCES = ["fa_api.cu", "fa_fwd.cu", "fa_bwd.cu", "fa_bwd_noalloc.cu", "fa_bwd_d256.cu", "fa_fwd_d256.cu", "fa_decode.cu", "fa_selftest.cu",
           "fa_fwd_fp8.cu"]
HEADERS = ["fa_internal.h", "fa_bwd_common.cuh", "fa_decode.h", "fa_fwd_fp8.h", "sm100.cuh", os.path.join("..", "..", "include", "fa.h")]


def nvcc() -> str:
    cand = [os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc"),
            shutil.which("nvcc") or ""]
    for c in cand:
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found (set CUDA_HOME)")


def flags() -> list[str]:
    return ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-Xptxas", "-v", "--expt-relaxed-constexpr"]


def _stale(so: str) -> bool:
    if not os.path.exists(so):
        return True
    t = os.path.getmtime(so)
    for f in SOURCES + HEADERS:
        if os.path.getmtime(os.path.join(CSRC, f)) > t:
            return True
    return False


def _build_one(so: str, extra: list[str], build_dir: str, verbose: bool) -> str:
    objs = []
    os.makedirs(build_dir, exist_ok=True)
    for src in SOURCES:
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *flags(), *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}")
        objs.append(obj)
    tmp = so + ".tmp"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs,
           "-Xcompiler", "-fPIC"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc link failed")
    os.replace(tmp, so)
    return so


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Builds libfa.so (and, unless debug=False, libfa_debug.so); returns libfa.so's path."""
    build_dir = os.path.join(HERE, "_build")
    if force or _stale(SO):
        _build_one(SO, [], build_dir, verbose)
    if debug and (force or _stale(SO_DEBUG)):
        _build_one(SO_DEBUG, ["-DFA_DEBUG"], os.path.join(build_dir, "debug"), verbose)
    return SO


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(SO)
