"""Build libpagedattn.so in-tree with nvcc for sm_100a (B200).

The kernels and their C ABI are one translation unit (csrc/pa_api.cu
includes the kernel headers); the host block manager is a second, plain C++
one. One nvcc call compiles and links both. The result lands next to
this file, where the binding loads it from.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libpagedattn.so")
SOURCES = [os.path.join(HERE, "csrc", "pa_api.cu"),
           os.path.join(HERE, "csrc", "pa_block_manager.cpp")]
DEPS = sorted(glob.glob(os.path.join(HERE, "csrc", "*")) +
              glob.glob(os.path.join(ROOT, "include", "*.h")))

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-o", LIB + ".tmp",
           *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


BENCH_BM = os.path.join(HERE, "pa_block_manager_bench")
BENCH_BM_SOURCES = [os.path.join(HERE, "csrc", "pa_block_manager_bench.cpp"),
                    os.path.join(HERE, "csrc", "pa_block_manager.cpp")]


def build_block_manager_bench(force: bool = False) -> str:
    """The host benchmark of the block manager (a plain C++ program)."""
    deps = BENCH_BM_SOURCES + [os.path.join(ROOT, "include", "pa_block_manager.h")]
    if (not force and os.path.exists(BENCH_BM) and
            all(os.path.getmtime(d) <= os.path.getmtime(BENCH_BM) for d in deps)):
        return BENCH_BM
    cxx = os.environ.get("CXX", "g++")
    cmd = [cxx, "-O2", "-std=c++17", "-I", os.path.join(ROOT, "include"), "-o", BENCH_BM + ".tmp",
           *BENCH_BM_SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(BENCH_BM + ".tmp", BENCH_BM)
    return BENCH_BM


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
