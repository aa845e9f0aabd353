"""Builds libsparge.so in-tree with nvcc for sm_100a (one translation unit)."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "sparge.cu")
HEADERS = [os.path.join(PKG, "csrc", f) for f in ("ptx.cuh", "mask.cuh", "attn.cuh", "linear.cuh", "lin_out.cuh", "lin_bwd.cuh", "quant.cuh", "attn_q8.cuh", "attn_bwd.cuh", "selftest.cuh")] + [
    os.path.join(ROOT, "include", "sparge.h")
]
LIB = os.path.join(PKG, "libsparge.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.exists(f) and os.path.getmtime(f) > t for f in [SRC, *HEADERS])


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), SRC, "-o", tmp]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.check_call(cmd, stdout=None if verbose else subprocess.DEVNULL)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
