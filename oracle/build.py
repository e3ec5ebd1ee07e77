"""Compile the CPU oracle (plain C, OpenMP) into oracle/liboracle.so.

Test infrastructure: only tests, the smoke check and the bench's CPU-baseline
leg load the result.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "crs_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

# -ffp-contract=off: the compiler must not fuse a*b+c on its own, so every
# rounding is the one the source spells out.
CFLAGS = ["-std=c11", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
          "-fvisibility=hidden"]


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", *CFLAGS, "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
