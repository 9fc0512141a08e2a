"""Build libpivot.so in-tree with nvcc for sm_100a (B200).

    python -m top_token_selection_b200.build [--force] [--debug]

Compiles every ``csrc/*.cu`` with relocatable device code (the per-device
error word is shared across translation units) and links one shared
library next to this file.  No GPU is needed to build.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libpivot.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-rdc=true", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-Wall", "-diag-suppress", "20044", f"-I{INCLUDE}"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(INCLUDE, "pivot.h"), __file__]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in _deps())


LIB_DEBUG = os.path.join(HERE, "libpivot_debug.so")


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build libpivot.so; with debug=True, libpivot_debug.so instead: the same
    sources with PIVOT_DEBUG defined, so every kernel checks its own index
    invariants and reports a failed check through the device error word
    (pivot_get_device_error returns PIVOT_ERR_DEVICE) instead of trapping."""
    lib = LIB_DEBUG if debug else LIB
    if not force and os.path.exists(lib) and \
            not any(os.path.getmtime(d) > os.path.getmtime(lib) for d in _deps()):
        return lib
    bdir = BUILD + ("_debug" if debug else "")
    os.makedirs(bdir, exist_ok=True)
    extra = ["-DPIVOT_DEBUG"] if debug else []
    objs = []
    for src in _sources():
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-rdc=true", "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
