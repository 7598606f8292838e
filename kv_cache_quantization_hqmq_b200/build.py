"""Builds libhqmq.so, the sm_100a CUDA library behind include/hqmq.h, in-tree.

    python -m kv_cache_quantization_hqmq_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libhqmq.so")
HEADER = os.path.join(ROOT, "include", "hqmq.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or verbose_ptxas or _stale():
        nvcc = os.environ.get("NVCC", "nvcc")
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [nvcc, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include")]
        if verbose_ptxas:
            cmd += ["-Xptxas", "-v"]
        cmd += sources() + ["-o", tmp]
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
