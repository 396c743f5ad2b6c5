"""Compile the CPU oracle (plain C) into ``oracle/liboracle.so``.

Test infrastructure only: the oracle is built so that the tests, the smoke check and
the benchmark's CPU-baseline leg can call it; the CUDA library never links it.

Flags: -O2 without any fast-math, with floating-point contraction off, so every
float operation in the oracle is the single IEEE operation its source line shows.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitlinear_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off",
          "-fexcess-precision=standard", "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)
            and os.path.getmtime(LIB) >= os.path.getmtime(__file__)):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
