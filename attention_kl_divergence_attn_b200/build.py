"""Builds libstreamkl.so (the C-ABI library) in-tree with nvcc for sm_100a.

Also builds libstreamkl_checked.so, the same library with every TMA coordinate
and global index checked against its tensor (STREAMKL_CHECK_BOUNDS): a debug
build for tests, which report an access outside a tensor through the status
word instead of faulting.

Usage: python -m attention_kl_divergence_attn_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libstreamkl.so")
CHECKED_LIB = os.path.join(PKG, "libstreamkl_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libstreamkl.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Builds libstreamkl.so, or with `checked` the bounds-checked debug build."""
    lib = CHECKED_LIB if checked else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + f".{os.getpid()}.tmp"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DSTREAMKL_CHECK_BOUNDS"] if checked else []), "-I", INCLUDE,
           os.path.join(CSRC, "streamkl.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build(force="--force" in sys.argv, checked=True))
