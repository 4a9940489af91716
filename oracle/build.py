"""Compile the CPU oracle (plain C++17, fp64) into oracle/liblcsa_oracle.so.

Test infrastructure: building the checker is allowed anywhere; running it is
reserved for the tests, the smoke check and the CPU-baseline benchmark leg.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lcsa_oracle.cpp")
LIB = os.path.join(HERE, "liblcsa_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-pthread", "-o", tmp, SRC]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
