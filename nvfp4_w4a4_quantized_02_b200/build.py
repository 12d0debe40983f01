"""Build the C-ABI shared library ``libnvfp4_w4a4.so`` in-tree with nvcc (sm_100a).

Usage: ``python -m nvfp4_w4a4_quantized_02_b200.build [--force]``.
The library is one translation unit (``csrc/nvfp4_api.cu``) that includes the
kernels; it links the CUDA runtime statically and needs no torch.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libnvfp4_w4a4.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
# The bounds-checking build: the same sources with -DNVFP4_DEBUG, in which every global
# store of the GEMM and quantiser kernels first checks its index invariants, records
# NVFP4_ERR_DEVICE_INDEX and skips the store when one fails.  Loaded by the Python
# binding when the environment sets NVFP4_DEBUG=1.
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libnvfp4_w4a4_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the NVFP4 library cannot be built")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(debug: bool = False) -> bool:
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile the library (``debug``: the bounds-checking build) if it is missing or
    older than its sources; return its path."""
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    if not force and not needs_build(debug):
        return path
    tmp = path + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, *(["-DNVFP4_DEBUG"] if debug else []), "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, os.path.join(CSRC, "nvfp4_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stdout + res.stderr)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
