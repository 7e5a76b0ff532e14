"""Build the CPU oracle (test infrastructure only) into oracle/libqlin_oracle.so.

Plain g++ with IEEE semantics: -O2 -ffp-contract=off -fno-fast-math, so every
float operation is the correctly rounded IEEE one and nothing is fused.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qlin_oracle.cpp")
LIB = os.path.join(HERE, "libqlin_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-pthread", SRC, "-o", LIB + ".tmp"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
