"""Builds the CPU oracle shared library (test infrastructure only).

    python oracle/build.py

Compiles mpzch_oracle.cpp with gcc at -O2, with floating-point contraction off
and without fast-math, so that its float arithmetic is plain IEEE binary32.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mpzch_oracle.cpp")
LIB = os.path.join(HERE, "libmpzch_oracle.so")
FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
         "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    deps = [SRC, os.path.join(HERE, "mpzch_oracle.h")]
    if not force and os.path.exists(LIB) and all(
            os.path.getmtime(LIB) >= os.path.getmtime(d) for d in deps):
        return LIB
    cmd = ["g++", *FLAGS, SRC, "-o", LIB]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
