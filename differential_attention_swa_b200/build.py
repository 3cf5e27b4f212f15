"""Builds libswa_attn.so in the package directory with nvcc for sm_100a.

The CUDA runtime is linked statically (nvcc's default), so the library does
not depend on which libcudart another component of the process loaded; the
driver API's tensor-map encoder is fetched at run time through the runtime,
so libcuda is not needed at link time either.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["api.cu", "prefill.cu", "decode.cu", "diff_decode.cu", "backward.cu"]
HEADERS = ["ptx.cuh", "schedule.cuh", "internal.h"]
LIB = os.path.join(HERE, "libswa_attn.so")
# Bounds-checking debug build: every TMA coordinate and global index checks
# itself (SWA_DEBUG_BOUNDS) and reports SWA_ERR_BOUNDS instead of accessing
# out of range. Used by the tests; never loaded by the release path.
LIB_DEBUG = os.path.join(HERE, "libswa_attn_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "swa_attn.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=(), debug_bounds: bool = False) -> str:
    """Compiles the library (or, with debug_bounds, its bounds-checking
    variant) if a source is newer than it; returns its path."""
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and not _stale(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    if not os.path.exists(nvcc) and os.path.exists("/usr/local/cuda/bin/nvcc"):
        nvcc = "/usr/local/cuda/bin/nvcc"
    flags = [*NVCC_FLAGS, *(["-DSWA_DEBUG_BOUNDS"] if debug_bounds else []), *extra]
    cmd = [nvcc, *flags, *[os.path.join(CSRC, s) for s in SOURCES], "-o", lib + ".tmp"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [],
          debug_bounds="--debug-bounds" in sys.argv)
