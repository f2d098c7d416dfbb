"""Build the CUDA library libfp8lin.so in-tree with nvcc for sm_100a.

    python fp8_block_scaled_12_b200/build.py [--force] [--verbose]

(run by path: importing the package loads the library this script builds)

The library is one translation unit (csrc/fp8lin.cu) compiled without fast-math
(IEEE division and rounding are part of the quantisers' contract) and linked
against the static CUDA runtime; it needs no GPU to build.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libfp8lin.so")
SOURCES = ["fp8lin.cu"]
DEPS = ["fp8lin.cu", "gemm.cuh", "gemm_mx.cuh", "gemm_swap.cuh", "moe.cuh", "quant.cuh", "ptx.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(ROOT, "include", "fp8lin.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "--shared", "-Xcompiler", "-fPIC", "-cudart", "static", "-I", os.path.join(ROOT, "include"),
           "-o", LIB] + [os.path.join(CSRC, s) for s in SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
