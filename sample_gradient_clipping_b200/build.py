"""Builds libdpclip.so in-tree for sm_100a with nvcc (no GPU needed: nvcc cross-compiles)."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdpclip.so")
# The same sources with -DDPCLIP_DEBUG: device-side index checks that record a failed check in
# the status word and skip the access (never a trap).
DEBUG_LIB = os.path.join(PKG, "libdpclip_debug.so")
SOURCES = [os.path.join(CSRC, "dpclip.cu")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    files = list(SOURCES)
    for d in (CSRC, INCLUDE):
        files += [os.path.join(d, f) for f in os.listdir(d) if f.endswith((".cuh", ".h", ".cu"))]
    return files


def up_to_date(path=LIB):
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(f) <= t for f in _deps())


def build(force=False, verbose=False, extra=(), debug=False):
    """Compile the library (or, with ``debug``, its checked variant) unless it is newer than
    every source; returns its path."""
    out = DEBUG_LIB if debug else LIB
    if not force and up_to_date(out):
        return out
    cmd = [_nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-I", CSRC, *(["-DDPCLIP_DEBUG"] if debug else []), *extra, "-o", out + ".tmp",
           *SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
