"""Build step of the CUDA library: nvcc for sm_100a into an in-tree shared object."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libwinattn.so")
DEBUG_LIB = os.path.join(HERE, "libwinattn_debug.so")
MAIN = os.path.join(HERE, "csrc", "winattn.cu")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++20",
              "-Xcompiler", "-fPIC", "-shared"]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu*")) +
                  glob.glob(os.path.join(ROOT, "include", "*.h")))


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """The library, or with debug=True its bounds-checking build (every token
    index and TMA box origin checked, violations reported through the device
    status word as WINATTN_ERR_DEVICE_BOUNDS)."""
    lib = DEBUG_LIB if debug else LIB
    if force or stale(lib):
        nvcc = os.environ.get("NVCC", "nvcc")
        cmd = [nvcc, *NVCC_FLAGS, *(["-DWINATTN_DEBUG"] if debug else []), "-o", lib, MAIN]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    build(force=True, verbose=True)
