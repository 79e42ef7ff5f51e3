"""Builds libmpzch.so (the sm_100a CUDA library) in-tree.

    python -m hashed_sparse_table_b200.build [--force]

nvcc compiles csrc/mpzch.cu for sm_100a only, without fast-math (the Writeback
and the int8 export rely on IEEE-rounded subtraction and division).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmpzch.so")
SOURCES = [os.path.join(CSRC, "mpzch.cu"), os.path.join(CSRC, "mpzch_res.cu")]
DEPS = SOURCES + [os.path.join(CSRC, "mpzch_kernels.cuh"), os.path.join(CSRC, "mpzch_tier.cuh"),
                  os.path.join(CSRC, "mpzch_internal.h"),
                  os.path.join(ROOT, "include", "mpzch.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-fmad=false", "-I", os.path.join(ROOT, "include")]


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and os.path.exists(LIB) and all(
            os.path.getmtime(LIB) >= os.path.getmtime(d) for d in DEPS):
        return LIB
    cmd = [NVCC, *FLAGS, *SOURCES, "-o", LIB + ".tmp"]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
