"""Compile the oracle's C code (the E4M3 and E5M2 codecs) into oracle/liboracle_fp8.so.

Test infrastructure only: see the package docstring.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRCS = [os.path.join(HERE, "e4m3.c"), os.path.join(HERE, "e5m2.c")]
LIB = os.path.join(HERE, "liboracle_fp8.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and all(os.path.getmtime(LIB) >= os.path.getmtime(s) for s in SRCS):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", *SRCS, "-o", LIB, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
