"""Build the CPU oracle (test infrastructure only) into oracle/liboracle.so.

Flags: -ffp-contract=off and no fast-math, so every product and sum in the C
source is one IEEE-754 round-to-nearest-even operation.  OpenMP only spreads
loops whose iterations each compute whole outputs sequentially (the integer
matmul's rows, the BitDelta and group-scale outputs), so results do not
depend on the thread count.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitnet_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fno-finite-math-only", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
