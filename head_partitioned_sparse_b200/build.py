"""Build libspa.so (sm_100a) in the package directory with nvcc.

Usage: python -m head_partitioned_sparse_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libspa.so")
SOURCES = ["spa_api.cu", "k_index_append.cu", "k_kv_append.cu", "k_select.cu", "k_attend.cu", "k_attend_mma.cu",
           "spa_noalloc.cu", "k_aoh.cu", "k_prefill_tc.cu", "k_cp.cu"]
HEADERS = ["spa_internal.cuh", os.path.join("..", "..", "include", "spa.h")]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    files = SOURCES + HEADERS + [os.path.basename(__file__)]
    dirs = [CSRC] * (len(SOURCES) + len(HEADERS)) + [PKG]
    return any(os.path.getmtime(os.path.join(d, f)) > t for d, f in zip(dirs, files))


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every CUDA source into libspa.so for sm_100a; returns the library path."""
    if not force and not _stale():
        return LIB
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "--shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", os.path.join(ROOT, "include"), "-o", LIB + ".tmp"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv))
