"""Compile the plain-C oracle (fk_oracle.c) into oracle/liboracle.so with gcc.

Test infrastructure only: the oracle is the checker for the CUDA library and
is never linked into it.  IEEE semantics are kept on purpose: no -ffast-math,
and floating-point contraction (a*b+c -> fma) is switched off so that every
operation rounds exactly as written in the C source.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fk_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-std=gnu11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]


def needs_build() -> bool:
    return (not os.path.exists(LIB)) or os.path.getmtime(LIB) < os.path.getmtime(SRC)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm", "-lpthread"]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)  # atomic: concurrent builders never see a partial file
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
