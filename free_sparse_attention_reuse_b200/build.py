"""Build the sm_100a CUDA library libmcs.so in-tree (nvcc; no GPU needed to compile)."""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmcs.so")
SOURCES = ["mcs_api.cu"]
DEPS = ["mcs_api.cu", "sm100.cuh", "attn.cuh", "select.cuh", "pddp.cuh", "variants.cuh", "kmeans.cuh"]
HEADER = os.path.join(os.path.dirname(HERE), "include", "mcs.h")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(verbose_ptxas: bool = False):
    f = [
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "--expt-relaxed-constexpr",
        "-Xcompiler", "-fPIC", "-shared",
        "-lcudart",
    ]
    if verbose_ptxas:
        f += ["-Xptxas", "-v"]
    return f


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, s) for s in DEPS] + [HEADER]
    return any(os.path.getmtime(s) > t for s in srcs)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not stale():
        return LIB
    cmd = [nvcc()] + flags(verbose_ptxas) + [os.path.join(CSRC, s) for s in SOURCES] + ["-o", LIB + ".tmp"]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError("nvcc failed building libmcs.so")
    if verbose_ptxas:
        sys.stderr.write(proc.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
