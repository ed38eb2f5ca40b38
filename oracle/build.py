"""Compile the oracle's C arithmetic (model.c) into liborc_model.so.

Test infrastructure only (see oracle/__init__.py).  Plain gcc, -O2 with
OpenMP; no fast-math, so the fp64 arithmetic stays IEEE.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "model.c")
LIB = os.path.join(HERE, "liborc_model.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, SRC, "-lm"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
