"""Builds libsolattn.so in-tree with nvcc for sm_100a (no GPU needed)."""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsolattn.so")
SOURCES = ["sol_attn_api.cu"]


def deps() -> list:
    """Every CUDA source and header under csrc/, so an edit to any of them rebuilds."""
    return sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def command(out: str = LIB, verbose_ptxas: bool = False) -> list:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", out]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    return cmd + [os.path.join(CSRC, s) for s in SOURCES]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    files = [os.path.join(CSRC, d) for d in deps()] + [os.path.join(ROOT, "include", "sol_attn.h")]
    return all(os.path.getmtime(d) <= t for d in files)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or not up_to_date():
        tmp = LIB + ".tmp"
        subprocess.run(command(tmp, verbose_ptxas), check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
