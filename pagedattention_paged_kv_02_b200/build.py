"""Build ``libpa.so`` in-tree with nvcc for sm_100a.

    python -m pagedattention_paged_kv_02_b200.build [--force] [--verbose]

The library is one translation unit (``csrc/pa_lib.cu``) compiled with
``-gencode arch=compute_100a,code=sm_100a``, the CUDA runtime linked
statically, and the C ABI of ``include/pa.h``.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libpa.so")
SRC = os.path.join(HERE, "csrc", "pa_lib.cu")


def _inputs():
    return (glob.glob(os.path.join(HERE, "csrc", "*")) +
            glob.glob(os.path.join(ROOT, "include", "*.h")))


def nvcc_command(out: str = LIB, verbose: bool = False):
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"),
           "-o", out, SRC]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library unless it is newer than every source."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in _inputs())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    tmp = LIB + ".tmp"
    subprocess.check_call(nvcc_command(tmp, verbose))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
