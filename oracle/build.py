"""Compile the C oracle (oracle.c) into liboracle.so next to this file.

Test infrastructure: the oracle is the plain CPU reference the CUDA library is
checked against.  Flags: -O2 for speed, -ffp-contract=off and no fast-math so
that every fp32 step is one IEEE operation, OpenMP for the loops over heads
and query rows (reductions inside a value stay sequential).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = [
    "-O2", "-std=c11", "-fPIC", "-shared",
    "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
    "-fopenmp", "-Wall", "-Wextra", "-Wno-unused-parameter",
]


def build(force: bool = False) -> str:
    """Build liboracle.so if it is missing or older than oracle.c; return its path."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)
            and os.path.getmtime(LIB) >= os.path.getmtime(__file__)):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
