"""Build the CUDA library liblnq.so in-tree for sm_100a (nvcc cross-compiles without a GPU)."""
from __future__ import annotations

import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_PATH = os.path.join(PKG, "liblnq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _inputs():
    return (sorted(glob.glob(os.path.join(CSRC, "*.cu")))
            + sorted(glob.glob(os.path.join(CSRC, "*.cuh")))
            + [os.path.join(ROOT, "include", "lnq.h"), os.path.abspath(__file__)])


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build_library(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ into liblnq.so (shared, position independent)."""
    if not force and not is_stale():
        return LIB_PATH
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [NVCC, *NVCC_FLAGS, "-shared", "-I", os.path.join(ROOT, "include"), *srcs, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    import sys
    print(build_library(force="--force" in sys.argv, verbose="-v" in sys.argv))
