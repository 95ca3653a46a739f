"""Compile the C++ oracle (moe_oracle.cpp -> libmoe_oracle.so) with g++.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  Run as
`python -m oracle.build`; __graft_entry__.build() also calls build().
-ffp-contract=off keeps each fp32 step of the pack a separately rounded
operation, as the format's definition requires.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
LIB = os.path.join(HERE, "libmoe_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
           SRC, "-o", LIB]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
