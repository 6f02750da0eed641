"""Builds libgqadecode.so in-tree with nvcc for sm_100a (B200), and its
checked twin libgqadecode_checked.so (-DGQA_CHECKED: index checks on the
kernels' derived global accesses, reported in the status word).

    python gqa_split_kv_decode_b200/_build.py [--verbose-ptxas]

Run it as a file (not with -m): importing the package loads the library it
builds.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libgqadecode.so")
LIB_CHECKED = os.path.join(PKG, "libgqadecode_checked.so")
SOURCES = [os.path.join(CSRC, "gqa_decode.cu")]
INCLUDE = os.path.join(ROOT, "include")
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-shared", "-cudart", "static",
    "-I", os.path.join(ROOT, "include"),
]


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, verbose_ptxas: bool = False, checked: bool = False) -> str:
    """Builds one of the two libraries (the normal one unless `checked`)."""
    lib = LIB_CHECKED if checked else LIB
    if not (force or stale(lib)):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *(["-DGQA_CHECKED"] if checked else []),
           *(["-Xptxas", "-v"] if verbose_ptxas else []), "-o", tmp, *SOURCES]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


def build_all(force: bool = False, verbose_ptxas: bool = False) -> list:
    return [build(force, verbose_ptxas), build(force, False, checked=True)]


if __name__ == "__main__":
    for path in build_all(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv):
        print(path)
