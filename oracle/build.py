"""Builds the C++ oracle (oracle/tokenbutler.cpp) into oracle/libtboracle.so
with the host compiler (fp64, OpenMP over independent rows).  Test
infrastructure: built by __graft_entry__.build() and on first use by
oracle/native.py; the product path never loads it."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "tokenbutler.cpp")
LIB = os.path.join(HERE, "libtboracle.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(SRC) > os.path.getmtime(LIB):
        # -ffp-contract=off: every product and sum rounds separately, in source order
        cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", SRC, "-o", LIB]
        print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force=True)
