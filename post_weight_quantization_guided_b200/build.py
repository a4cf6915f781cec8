"""Build the CUDA library liblnq.so in-tree for sm_100a (nvcc cross-compiles without a GPU).

Each translation unit under csrc/ is compiled to its own object (in parallel, under _build/ at the
repository root), then the objects are linked into one shared library.
"""
from __future__ import annotations

import glob
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(PKG, "liblnq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _shared_inputs():
    """Files every translation unit depends on: the headers and this script."""
    return (sorted(glob.glob(os.path.join(CSRC, "*.cuh")))
            + [os.path.join(ROOT, "include", "lnq.h"), os.path.abspath(__file__)])


def _obj(src: str) -> str:
    return os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + ".o")


def _newest(paths) -> float:
    return max(os.path.getmtime(p) for p in paths)


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    return _newest(_sources() + _shared_inputs()) > os.path.getmtime(LIB_PATH)


def _compile(src: str, force: bool, verbose: bool) -> str:
    obj = _obj(src)
    if (not force and os.path.exists(obj)
            and os.path.getmtime(obj) >= _newest([src] + _shared_inputs())):
        return obj
    tmp = obj + f".tmp{os.getpid()}"
    cmd = [NVCC, *NVCC_FLAGS, "-c", "-I", os.path.join(ROOT, "include"), src, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, obj)
    return obj


def build_library(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ and link liblnq.so (shared, position independent)."""
    if not force and not is_stale():
        return LIB_PATH
    os.makedirs(OBJ_DIR, exist_ok=True)
    srcs = _sources()
    with ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 4)) as pool:
        objs = list(pool.map(lambda s: _compile(s, force, verbose), srcs))
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           *objs, "-o", tmp])
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    import sys
    print(build_library(force="--force" in sys.argv, verbose="-v" in sys.argv))
