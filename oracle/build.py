"""Compile the fp64 C oracle into ``oracle/liboracle_specverify.so``.

Test infrastructure: the oracle is built so that the test suite, the smoke
check and the benchmark's CPU-baseline leg can call it.  Plain ``gcc -O2``
with floating-point contraction off, so every fp64 operation rounds exactly
as written in the source.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "specverify_oracle.c")
LIB = os.path.join(HERE, "liboracle_specverify.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
