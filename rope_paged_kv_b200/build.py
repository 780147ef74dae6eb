"""Build ``librope_store.so`` (the C-ABI library of include/rope_store.h) for sm_100a.

    python rope_paged_kv_b200/build.py [--force]

Run it as a script, or load it from its file: importing the package itself needs the built
library, so the builder must not be reached through the package.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "librope_store.so")
SOURCES = [os.path.join(CSRC, "rope_store.cu")]
HEADERS = ["device_utils.cuh", "pipeline.cuh", "common.cuh", "banded.cuh", "bshd.cuh", "radd.cuh",
           "gemv_norm.cuh"]
DEPS = SOURCES + [os.path.join(CSRC, h) for h in HEADERS] + [
                  os.path.join(ROOT, "include", "rope_store.h")]

NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-Xcompiler", "-fPIC", "-shared", "-Xcompiler", "-Wall"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or older than its sources; return its path."""
    if not force and not stale():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc()] + NVCC_FLAGS + ["-I", os.path.join(ROOT, "include"), "-o", tmp] + SOURCES
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
