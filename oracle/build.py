"""Compile the fp64 CPU oracle (test infrastructure) into oracle/liboracle_swin.so.

Plain C99 + OpenMP, built with gcc. Nothing in the GPU library links or
includes it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "swin_oracle.c")
LIB = os.path.join(HERE, "liboracle_swin.so")


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-std=c99", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
