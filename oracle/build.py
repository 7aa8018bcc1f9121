"""Compile the fp64 CPU oracle into oracle/libspin_oracle.so.

The oracle is test infrastructure: only the test suite, the smoke check and
the CPU-baseline leg of the benchmark load it.  It is plain C built with gcc,
with strict IEEE semantics (no fast-math, no FMA contraction), so that every
operation it performs is the correctly rounded binary64 operation written in
the source. OpenMP only spreads independent rows of the batch loop over
threads.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "spin_oracle.c")
LIB = os.path.join(HERE, "libspin_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
           "-frounding-math", "-fopenmp", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
