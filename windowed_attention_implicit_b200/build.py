"""Builds librib.so in-tree for sm_100a with nvcc.

    python -m windowed_attention_implicit_b200.build
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
LIB = os.path.join(PKG, "librib.so")
# the same library with every non-TMA global access bounds-checked (RIB_DEBUG)
LIB_DEBUG = os.path.join(PKG, "librib_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh"))) + [os.path.join(INCLUDE, "rib.h")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compiles librib.so (or, with debug=True, librib_debug.so: the same
    sources with RIB_DEBUG, every non-TMA global access bounds-checked)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DRIB_DEBUG"] if debug else []), "-I", INCLUDE, "-o", tmp,
           os.path.join(CSRC, "rib.cu")]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
