"""Builds libdash_attn.so in-tree (sm_100a, no GPU needed to compile).

    python -m persistent_sm_attn_b200.build [--force] [--ptxas-verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdash_attn.so")
SOURCES = ["dash_api.cu", "noalloc.cu", "sched.cpp"]
DEPS = SOURCES + ["sched.h", "internal.h", "ptx.cuh", "bwd_kernel.cuh", "fwd_kernel.cuh",
                  "aux_kernels.cuh"]
HEADER = os.path.join(os.path.dirname(HERE), "include", "dash_attn.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2", "-shared",
]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    files = [os.path.join(CSRC, f) for f in DEPS] + [HEADER]
    return any(os.path.getmtime(f) > t for f in files)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not _stale():
        return LIB
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    cmd = [nvcc, *NVCC_FLAGS]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES] + ["-o", LIB + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="--ptxas-verbose" in sys.argv)
    print(LIB)
