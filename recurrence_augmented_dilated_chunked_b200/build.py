"""Build the in-tree CUDA library ``libratp.so`` for sm_100a with nvcc.

``python -m recurrence_augmented_dilated_chunked_b200.build`` (or
``build_library()``) compiles ``csrc/ratp.cu`` with
``-gencode arch=compute_100a,code=sm_100a``; nvcc cross-compiles, so no GPU is
needed.  The shared library lands next to this file, where the Python binding
loads it.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libratp.so")
# guarded debug build: every kernel-addressed global access range-checked
GUARDED_LIB = os.path.join(PKG, "libratp_guarded.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-O3", "-std=c++17", "-lineinfo", "--use_fast_math",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "-I", INCLUDE, "-I", CSRC,
]


def _sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))] + \
        [os.path.join(INCLUDE, f) for f in sorted(os.listdir(INCLUDE))]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in _sources())


def build_library(force: bool = False, verbose: bool = False, extra=(), guarded: bool = False) -> str:
    """Compile ``libratp.so`` (or, guarded=True, ``libratp_guarded.so`` with
    -DRATP_GUARDED) unless it is newer than every source."""
    lib = GUARDED_LIB if guarded else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    flags = FLAGS + (["-DRATP_GUARDED"] if guarded else [])
    cmd = [NVCC] + flags + list(extra) + ["-o", tmp, os.path.join(CSRC, "ratp.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    verbose = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    print(build_library(force=True, verbose=verbose, extra=extra, guarded="--guarded" in sys.argv))
