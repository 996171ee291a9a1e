"""Builds the in-tree CUDA library ``libkivi.so`` (sm_100a) with nvcc.

    python -m bit_asymmetric_kv_02_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libkivi.so")
LIB_DEBUG = os.path.join(PKG, "libkivi_debug.so")   # -DKIVI_DEBUG: device-side bounds checks
SOURCES = ["kivi_api.cu", "quantize.cu", "decode.cu", "noalloc.cu"]
HEADERS = ["common.cuh", "kernels.h", "quant_rules.cuh"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put CUDA's bin/ on PATH")


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "kivi.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    """Compiles libkivi.so next to this file (skipped when up to date) and returns its path.
    debug=True builds libkivi_debug.so instead, with -DKIVI_DEBUG (the kernels' bounds checks)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not verbose_ptxas and not _stale(lib):
        return lib
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC, "-o", lib + ".tmp"]
    if debug:
        cmd += ["-DKIVI_DEBUG"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + proc.stdout + proc.stderr)
    if verbose_ptxas:
        sys.stderr.write(proc.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv, debug="--debug" in sys.argv))
