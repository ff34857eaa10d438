"""Build libmilo.so in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmilo.so")
TRACE_LIB = os.path.join(PKG, "libmilo_trace.so")   # decode timeline build (-DMILO_DECODE_TRACE)

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(INCLUDE, "milo.h")])


def build(force: bool = False, verbose: bool = False, extra=(), trace: bool = False) -> str:
    """Build libmilo.so (or, with `trace`, libmilo_trace.so: the same library
    whose decode kernel records a per-warp timeline) if a source is newer."""
    lib = TRACE_LIB if trace else LIB
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= newest and not extra:
        return lib
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    flags = [*NVCC_FLAGS, *(["-DMILO_DECODE_TRACE"] if trace else []), *extra]
    cmd = [nvcc, *flags, "-I", INCLUDE, "-I", CSRC, "-o", tmp, os.path.join(CSRC, "milo.cu"), "-lcudart"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, trace="--trace" in sys.argv,
                extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else []))
