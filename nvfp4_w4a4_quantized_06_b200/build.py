"""Build the sm_100a C-ABI library in-tree: libnvfp4w4a4.so next to this file.

    python -m nvfp4_w4a4_quantized_06_b200.build
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnvfp4w4a4.so")
SOURCES = [os.path.join(CSRC, "nvfp4w4a4.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("ptx.cuh", "quantize.cuh", "gemm.cuh", "gemm_pair.cuh", "gemm_cluster.cuh")] + [
    os.path.join(ROOT, "include", "nvfp4w4a4.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def command(out: str = LIB, verbose_ptxas: bool = False) -> list[str]:
    cmd = [nvcc(), "-std=c++17", "-O3", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "--expt-relaxed-constexpr", "-o", out] + SOURCES
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or stale():
        tmp = LIB + ".tmp"
        subprocess.run(command(tmp, verbose_ptxas), check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
