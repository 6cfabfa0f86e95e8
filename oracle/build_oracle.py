"""Builds the CPU oracle (TEST INFRASTRUCTURE ONLY) into oracle/liboracle.so with g++.

The oracle is plain C++17 with no CUDA; it is compiled without floating-point contraction so
that every product and sum rounds as written.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "liboracle.so")
SRCS = [os.path.join(HERE, "gs_oracle.cpp")]
DEPS = SRCS + [os.path.join(HERE, "gs_oracle.hpp")]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in DEPS)
        if os.path.getmtime(LIB) >= newest:
            return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-pthread", "-Wall", "-o", tmp] + SRCS
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
