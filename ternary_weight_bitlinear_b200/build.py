"""Build libbitlinear.so (the C-ABI library of CUDA kernels) for sm_100a, in-tree.

    python -m ternary_weight_bitlinear_b200.build [--force] [--verbose]
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libbitlinear.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-I" + INCLUDE, "-I" + CSRC,
         "-Xcompiler", "-Wall", "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "bitlinear.h")])


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ into libbitlinear.so when stale; return its path."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(f) for f in sources())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cus = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, *cus]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
