"""Ahead-of-time build of the CUDA library (sm_100a) into this package folder.

    python sparse_attention_indexer_strided_b200/build.py [--force] [-v]

Run it as a script (or load it by file path): the package itself cannot be
imported before the library exists.

nvcc cross-compiles without a GPU. The shared object keeps every symbol hidden
except the C ABI declared in include/dsa_topk.h.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "dsa_topk.cu")
HDR = os.path.join(ROOT, "include", "dsa_topk.h")
LIB = os.path.join(PKG, "libdsa_topk.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    csrc = os.path.dirname(SRC)
    deps = [HDR] + [os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh", ".h"))]
    stale = not os.path.exists(LIB) or any(os.path.getmtime(p) > os.path.getmtime(LIB) for p in deps)
    if force or stale:
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [nvcc()] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose else []) + [
            "-I" + os.path.join(ROOT, "include"), SRC, "-o", tmp]
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
