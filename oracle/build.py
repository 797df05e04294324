"""Build the CPU oracle (plain C, gcc, OpenMP) into oracle/libdg_oracle.so.

Test infrastructure: the oracle is only ever loaded by the test suite, the smoke
check and the CPU-baseline leg of the benchmark.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dg_oracle.c")
LIB = os.path.join(HERE, "libdg_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    # no -ffast-math: the oracle relies on IEEE double arithmetic and SSE2 evaluation
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
           "-fno-fast-math", "-ffp-contract=off", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
