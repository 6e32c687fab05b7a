"""Builds libblasst.so (the C-ABI library of include/blasst.h) for sm_100a.

    python dynamic_block_sparse_fa_b200/build.py [--force] [--verbose]

The library is one nvcc translation unit (csrc/blasst.cu) compiled for
sm_100a with the CUDA runtime linked statically; it lands next to this file
so that it travels with the source tree.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libblasst.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _sources():
    files = [os.path.join(INCLUDE, "blasst.h")]
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            files.append(os.path.join(CSRC, name))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if a source is newer than it; returns its path."""
    if not force and up_to_date():
        return LIB
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
           "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-I", CSRC, "-o", LIB,
           os.path.join(CSRC, "blasst.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
