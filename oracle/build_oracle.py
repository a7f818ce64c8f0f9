"""Compile the CPU oracle (aq_oracle.cpp) into oracle/libaq_oracle.so.

Test infrastructure only.  Flags keep fp32 arithmetic IEEE-exact: no FMA
contraction and no fast-math, so the quantizer's codes are the ones its
definition fixes.  OpenMP parallelises only the independent output rows of the
matmul and conv references.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "aq_oracle.cpp")
LIB = os.path.join(HERE, "libaq_oracle.so")

FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
         "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.run(["g++", *FLAGS, SRC, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
