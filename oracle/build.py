"""Compile the fp64 C oracle into oracle/libkda_oracle.so.

Test infrastructure only: this builds the oracle library that tests/, smoke() and the
CPU-baseline leg of bench.py load; nothing in the product links it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kda_oracle.c")
LIB = os.path.join(HERE, "libkda_oracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    # Plain -O2, no -ffast-math and no -march: IEEE fp64 on any x86-64 host.
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99",
           "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
