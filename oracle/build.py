"""Compile the fp64 CPU oracle (oracle/gret_oracle.c) into oracle/libgret_oracle.so.

Test infrastructure: the oracle is built here so that the tests, the smoke check and the
benchmark's CPU-baseline leg can call it.  Nothing in the CUDA library uses it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gret_oracle.c")
LIB = os.path.join(HERE, "libgret_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
