"""Build the CUDA library libinfini_attn.so in-tree for sm_100a.

    python -m compressive_memory_segment_b200.build [--force] [--trace | --debug] [--ptxas-v]

nvcc compiles for sm_100a only (-gencode arch=compute_100a,code=sm_100a) with
line info for the profiler; the CUDA runtime is linked statically so the
library needs nothing at load time beyond the driver. The driver API entry
point used to encode TMA tensor maps is fetched at run time through the
runtime, so libcuda is not linked either.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libinfini_attn.so")
# Tracing build: the same library with INFINI_TRACE defined (clock64 records of
# the paired attention kernel's pipeline on CTA 0; include/infini_attn_trace.h).
TRACE_LIB = os.path.join(LIBDIR, "libinfini_attn_trace.so")
# Debug build: the same library with INFINI_DEBUG defined (device-side index
# checks that record INFINI_ERR_BOUNDS in the status word instead of trapping).
DEBUG_LIB = os.path.join(LIBDIR, "libinfini_attn_debug.so")
MAIN = os.path.join(CSRC, "infini_attn.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def _sources():
    return [MAIN] + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False, extra=None, trace: bool = False,
          debug: bool = False) -> str:
    """Compile libinfini_attn.so (or, with trace=True, the tracing build
    libinfini_attn_trace.so; with debug=True, the index-checking build
    libinfini_attn_debug.so) unless it is newer than every source."""
    os.makedirs(LIBDIR, exist_ok=True)
    lib = TRACE_LIB if trace else (DEBUG_LIB if debug else LIB)
    if not force and os.path.exists(lib):
        t = os.path.getmtime(lib)
        if all(os.path.getmtime(s) <= t for s in _sources()):
            return lib
    tmp = lib + ".tmp%d" % os.getpid()
    flags = list(extra or []) + (["-DINFINI_TRACE"] if trace else []) + (["-DINFINI_DEBUG"] if debug else [])
    cmd = [nvcc(), *NVCC_FLAGS, *flags, "-I", os.path.join(ROOT, "include"), MAIN, "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, trace="--trace" in sys.argv, debug="--debug" in sys.argv,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None))
