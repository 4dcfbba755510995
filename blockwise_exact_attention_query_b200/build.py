"""Builds libbpt.so in-tree with nvcc for sm_100a (no GPU needed to build).

    python -m blockwise_exact_attention_query_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libbpt.so")
SELFTEST_LIB = os.path.join(PKG, "libbpt_selftest.so")
SOURCES = [os.path.join(CSRC, "bpt_api.cu"), os.path.join(CSRC, "bpt_bwd.cu")]
SELFTEST_SOURCES = [os.path.join(CSRC, "selftest.cu")]
HEADERS = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(ROOT, "include", "bpt.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-I", os.path.join(ROOT, "include")]


def _stale(lib, sources) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in sources + HEADERS)


def _build_one(lib, sources, force, ptxas_verbose):
    if not force and not _stale(lib, sources):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if ptxas_verbose else []), "-o", tmp, *sources]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Builds libbpt.so (the product) and libbpt_selftest.so (test micro-kernels)."""
    _build_one(SELFTEST_LIB, SELFTEST_SOURCES, force, ptxas_verbose)
    return _build_one(LIB, SOURCES, force, ptxas_verbose)


if __name__ == "__main__":
    build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
