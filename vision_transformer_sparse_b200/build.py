"""Build the in-tree C-ABI library `libbra.so` for sm_100a with nvcc.

    python -m vision_transformer_sparse_b200.build          # build if stale
    python -m vision_transformer_sparse_b200.build --force  # rebuild
    python -m vision_transformer_sparse_b200.build --ptxas  # print register/smem use

The library is built next to this file so that it travels with the source tree;
nothing is installed into site-packages.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libbra.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-shared",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "bra.h"), os.path.abspath(__file__)]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _deps())


def build_library(force: bool = False, verbose: bool = False, ptxas: bool = False) -> str:
    if not (force or ptxas or stale()):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [NVCC] + ARCH + FLAGS + (["-Xptxas", "-v"] if ptxas else []) + ["-o", tmp] + _sources()
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if ptxas:
        print(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build_library(force="--force" in sys.argv, verbose=True, ptxas="--ptxas" in sys.argv)
    print(LIB)
