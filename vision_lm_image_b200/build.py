"""Builds the CUDA library in-tree: vision_lm_image_b200/libmimo_b200.so (sm_100a).

    python -m vision_lm_image_b200.build [--force] [--checked]

nvcc cross-compiles for sm_100a without a GPU. The build is skipped when the
shared object is newer than every source file.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libmimo_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
# debug build whose pixel kernels check every global access (include/mimo.h, mimo_bounds_check_status)
CHECKED_LIB_PATH = os.path.join(PKG, "libmimo_b200_checked.so")
CHECKED_FLAGS = ["-DMIMO_BOUNDS_CHECK"]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _inputs() -> list[str]:
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None, out: str = LIB_PATH) -> str:
    if not force and up_to_date(out):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "--shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-Wall", "-I", INCLUDE, "-I", CSRC, *sources(), "-o", tmp, *(extra or [])]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build_checked(force: bool = False, verbose: bool = False) -> str:
    """The bounds-checked debug build (a separate shared object beside the release one)."""
    return build(force=force, verbose=verbose, extra=CHECKED_FLAGS, out=CHECKED_LIB_PATH)


if __name__ == "__main__":
    if "--checked" in sys.argv:
        print(build_checked(force="--force" in sys.argv, verbose=True))
    else:
        build(force="--force" in sys.argv, verbose=True,
              extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
        print(LIB_PATH)
