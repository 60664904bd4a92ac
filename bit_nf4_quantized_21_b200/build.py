"""Build libqlora.so in-tree for sm_100a with nvcc, and its debug build
libqlora_debug.so (-DQLORA_DEBUG_CHECKS: index-range checks in the kernels).

    python -m bit_nf4_quantized_21_b200.build        # rebuild when sources changed
    python -m bit_nf4_quantized_21_b200.build -v     # also print ptxas resource usage
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqlora.so")
LIB_DEBUG = os.path.join(PKG, "libqlora_debug.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not needs_build(lib) and not verbose:
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".{os.getpid()}.tmp"
    cmd = [nvcc, *NVCC_FLAGS, *(["-DQLORA_DEBUG_CHECKS"] if debug else []), "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, os.path.join(CSRC, "qlora.cu")]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
    print(build(force=True, debug=True))
