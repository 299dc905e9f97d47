"""CPU oracle for the strided indexer top-k -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import this package. The product library never does, and
this package imports nothing from it.

The oracle is the plain definition (see ``dsa_topk_oracle.cpp``): for each row,
a stable sort of the valid prefix ``[0, L_r)`` by value descending (ties keep
ascending index order), the first ``min(k, L_r)`` indices, then ``-1`` padding.
Row r starts at ``r * row_stride`` (vLLM PR #42169, "实现拆解": stride(0), not
size(1)).

Parity status: pinned (tests/test_oracle.py) by O(L^2) brute-force ranking,
exhaustive special values, NumPy / PyTorch stable sorts, closed forms and
invariants. The pages print no worked top-k example, so nothing is pinned to
printed output values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_topk_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with the host C++ compiler (plain -O2, no -ffast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_dsa_topk.restype = ctypes.c_int
        lib.oracle_dsa_topk.argtypes = [
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
            ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
        ]
        lib.oracle_hardware_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def hardware_threads() -> int:
    return int(_load().oracle_hardware_threads())


def topk(logits: np.ndarray, lengths: np.ndarray, k: int, threads: int = 0,
         row_stride: Optional[int] = None) -> np.ndarray:
    """Top-k indices per row. ``logits`` is float32, 2-D ``[rows, row_stride]``
    (C-contiguous) or 1-D flat with an explicit ``row_stride``. Returns int32
    ``[rows, k]``."""
    lib = _load()
    a = np.ascontiguousarray(logits, dtype=np.float32)
    L = np.ascontiguousarray(lengths, dtype=np.int32)
    if a.ndim == 2:
        rows, stride = a.shape
        if row_stride is not None and row_stride != stride:
            raise ValueError("row_stride disagrees with the 2-D shape")
    else:
        if row_stride is None:
            raise ValueError("flat logits need row_stride")
        stride = int(row_stride)
        rows = L.shape[0]
        if rows and a.size < (rows - 1) * stride + 1:
            raise ValueError("flat buffer too small")
    if L.shape[0] != rows:
        raise ValueError("lengths must have one entry per row")
    out = np.empty((rows, k), dtype=np.int32)
    rc = lib.oracle_dsa_topk(a.ctypes.data, stride, L.ctypes.data, rows, int(k),
                             out.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments (rc=%d)" % rc)
    return out
