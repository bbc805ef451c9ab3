"""Build libw8a8.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

    python w8a8_linear_layers_b200/build.py [--verbose] [--debug]

(--debug builds libw8a8_debug.so: the same kernels compiled with -DW8A8_DEBUG,
which count non-finite inputs and failed index checks for sq_debug_status.)

(Run it by path, or load it with importlib by path: importing the package
itself loads libw8a8.so, which is what this script produces.)

Flags: IEEE division/sqrt, no flush-to-zero, no FMA contraction (the kernels
write their fused multiply-adds explicitly), -lineinfo for profiling.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libw8a8.so")
LIB_DEBUG = os.path.join(PKG, "libw8a8_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "--fmad=false", "-I" + os.path.join(ROOT, "include"), "-I" + CSRC,
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(ROOT, "include", "w8a8.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def load_build_module():
    """This module, loaded by file path without importing the package."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("w8a8_build", os.path.abspath(__file__))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every kernel source into libw8a8.so (debug: libw8a8_debug.so
    with -DW8A8_DEBUG); returns its path."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [NVCC, *NVCC_FLAGS, *(["-DW8A8_DEBUG"] if debug else []), *(["-Xptxas", "-v"] if verbose else []),
           *sources(), "-o", tmp, "-lcudart"]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
