"""Compile the C oracle into ``oracle/librope_oracle.so`` (test infrastructure only).

Built with plain gcc, no fast-math and no floating-point contraction, so every double
operation in the oracle is an individually rounded IEEE operation.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "rope_oracle.c")
HDR = os.path.join(HERE, "rope_oracle.h")
LIB = os.path.join(HERE, "librope_oracle.so")


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its sources; return its path."""
    if not force and os.path.exists(LIB):
        lib_t = os.path.getmtime(LIB)
        if lib_t >= os.path.getmtime(SRC) and lib_t >= os.path.getmtime(HDR):
            return LIB
    tmp = LIB + ".tmp"
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC",
           "-shared", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
