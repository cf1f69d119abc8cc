"""Build the in-tree CUDA library (libqlora_nf4.so) for sm_100a with nvcc.

The library is one translation unit (csrc/qlora_api.cu includes the kernel
headers), compiled with IEEE division and denormal support (no fast math):
the quantizer's codes depend on correctly rounded fp32 division.

`--debug` builds the checked library (libqlora_nf4_debug.so, QLORA_DEBUG):
the same kernels with bounds and alignment checks before every TMA copy and
cluster exchange (include/qlora_nf4.h, qlora_debug_record).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqlora_nf4.so")
LIB_DEBUG = os.path.join(PKG, "libqlora_nf4_debug.so")
SOURCES = [os.path.join(CSRC, "qlora_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(INCLUDE, "qlora_nf4.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False, extra=None, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not needs_build(lib):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    flags = NVCC_FLAGS + (["-DQLORA_DEBUG"] if debug else [])
    cmd = [nvcc(), *flags, "-I", INCLUDE, "-I", CSRC, *(extra or []), "-o", tmp, *SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
