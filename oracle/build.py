"""Compile the host oracle (oracle.cpp) into liboracle.so beside it.

Plain g++, no fast-math and no FMA contraction, so every fp32 step of the
quantizer rounds once as IEEE specifies. Test infrastructure only.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")
FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
         "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(src: str = SRC, out: str = LIB, extra=()) -> str:
    cmd = ["g++", *FLAGS, *extra, src, "-o", out]
    subprocess.run(cmd, check=True)
    return out


def stale(src: str = SRC, out: str = LIB) -> bool:
    return not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src)


if __name__ == "__main__":
    print(build(*sys.argv[1:2]))
