"""Build libq4dec.so in-tree with nvcc for sm_100a, and beside it
libq4dec_debug.so: the same sources with Q4D_DEBUG defined (every global
access of every kernel index-checked into the device error record).

Usage: ``python -m bit_weight_streaming_dequant_b200.build`` (or
``__graft_entry__.build()``).  The libraries link the CUDA runtime
statically, so loading them needs no CUDA library path; they only need the
NVIDIA driver once a compute entry point is called.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libq4dec.so")
LIB_DEBUG = os.path.join(PKG, "libq4dec_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libq4dec")
    return path


def _compile(out: str, flags, verbose: bool):
    srcs = [os.path.join(CSRC, "q4dec.cu"), os.path.join(CSRC, "q4d_selftest.cu")]
    cmd = [nvcc(), *NVCC_FLAGS, *flags, "-I", INCLUDE, "-I", CSRC, *srcs, "-o", out + ".tmp"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)


def build(verbose: bool = False, extra_flags=None, debug: bool = True) -> str:
    """Compile the release library (and, with `debug`, the debug one)."""
    _compile(LIB, list(extra_flags or []), verbose)
    if debug:
        _compile(LIB_DEBUG, ["-DQ4D_DEBUG", *(extra_flags or [])], verbose)
    return LIB


if __name__ == "__main__":
    build(verbose=True, extra_flags=sys.argv[1:])
