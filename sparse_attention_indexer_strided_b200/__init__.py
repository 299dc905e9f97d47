"""Strided indexer top-k on B200: thin Python binding over the C ABI.

The work happens in ``libdsa_topk.so`` (hand-written sm_100a kernels); this
module only marshals torch tensors into the pointers, sizes and stream handle
that ``dsa_topk`` takes. There is no fallback: if the library is missing the
import fails.

Row addressing follows the stride fix in the vLLM PR #42169 report ("实现拆解"):
row r of ``logits`` starts at ``r * logits.stride(0)``, which may exceed the
valid length because the DeepGEMM logits are padded and sliced.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa_topk.so")
MAX_K = 2048

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libdsa_topk.so is not built; run `python sparse_attention_indexer_strided_b200/build.py` "
        "(nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32

_lib.dsa_topk.restype = ctypes.c_int
_lib.dsa_topk.argtypes = [_P, _I64, _P, _I64, _I32, _P, _P]
_lib.dsa_topk_ex.restype = ctypes.c_int
_lib.dsa_topk_ex.argtypes = [_P, _I32, _I64, _P, _I64, _I32, ctypes.c_uint32, _P, _I64, _P, _P]
_lib.dsa_topk_host.restype = ctypes.c_int
_lib.dsa_topk_host.argtypes = [_P, _I64, _P, _I64, _I32, _P, _P, _P, _P, _P]
_lib.dsa_topk_plan.restype = ctypes.c_int
_lib.dsa_topk_plan.argtypes = [_I64, _I64, _I32, ctypes.POINTER(_I32), ctypes.POINTER(_I32)]
_lib.dsa_topk_device_status.restype = ctypes.c_int
_lib.dsa_topk_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
_lib.dsa_topk_strerror.restype = ctypes.c_char_p
_lib.dsa_topk_strerror.argtypes = [ctypes.c_int]
_lib.dsa_topk_version.restype = ctypes.c_int
_lib.dsa_topk_version.argtypes = []
_lib.dsa_topk_set_test_hooks.restype = ctypes.c_int
_lib.dsa_topk_set_test_hooks.argtypes = [ctypes.c_uint64, _I64]

DTYPE_F32, DTYPE_BF16, DTYPE_F16 = 0, 1, 2
FLAG_UNSORTED = 1
_DTYPES = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}

STATUS_WAIT_TIMEOUT = 1
STATUS_SELECT_BROKEN = 2
STATUS_REREAD = 4
STATUS_ERRORS = STATUS_WAIT_TIMEOUT | STATUS_SELECT_BROKEN

lib = _lib  # raw ctypes handle, for callers that pass their own pointers


class DsaTopkError(RuntimeError):
    def __init__(self, code: int):
        super().__init__("dsa_topk failed (%d): %s" % (code, strerror(code)))
        self.code = code


def strerror(code: int) -> str:
    return _lib.dsa_topk_strerror(int(code)).decode()


def version() -> int:
    return int(_lib.dsa_topk_version())


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check_rows(logits: torch.Tensor, lengths: torch.Tensor, k: int, dtypes=(torch.float32,)) -> Tuple[int, int]:
    if logits.dtype not in dtypes or logits.dim() != 2:
        raise TypeError("logits must be a 2-D tensor of one of %s" % (dtypes,))
    if logits.size(0) > 0 and logits.size(1) > 1 and logits.stride(1) != 1:
        raise ValueError("logits rows must be contiguous along dim 1 (stride(1) == 1)")
    if lengths.dtype != torch.int32 or lengths.dim() != 1 or lengths.size(0) != logits.size(0):
        raise TypeError("lengths must be int32 [num_rows]")
    if not lengths.is_contiguous():
        raise ValueError("lengths must be contiguous")
    if not (1 <= int(k) <= MAX_K):
        raise ValueError("k must be in [1, %d]" % MAX_K)
    rows = int(logits.size(0))
    # the row stride, not the logical width (the stride(0)-vs-size(1) fix); a
    # 1-row view's stride(0) is never used to step rows, only to clamp lengths
    stride = int(logits.stride(0))
    if rows <= 1:
        stride = max(stride, int(logits.size(1)), 1)
    return rows, stride


def dsa_topk(logits: torch.Tensor, lengths: torch.Tensor, k: int,
             out: Optional[torch.Tensor] = None, stream=None, unsorted: bool = False,
             index_table: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Top-k row-local indices of ``logits[r, :lengths[r]]`` per row.

    ``logits``: CUDA float32, bfloat16 or float16 ``[num_rows, >= max L]``,
    any row stride. ``lengths``: CUDA int32 ``[num_rows]`` (clamped to [0,
    stride] on device). Returns (or fills ``out``) int32 ``[num_rows, k]``:
    value descending, ties by ascending index, -1 past ``min(k, L_r)``.
    ``unsorted``: the same index set per row, in unspecified order.
    ``index_table``: CUDA int32 ``[num_rows, >= max L]`` (any row stride); each
    selected index j of row r is written as ``index_table[r, j]``.
    Asynchronous on ``stream``.
    """
    rows, stride = _check_rows(logits, lengths, k, tuple(_DTYPES))
    if not (logits.is_cuda and lengths.is_cuda):
        raise ValueError("logits and lengths must be CUDA tensors (use dsa_topk_host for host buffers)")
    if out is None:
        out = torch.empty((rows, k), dtype=torch.int32, device=logits.device)
    elif out.dtype != torch.int32 or tuple(out.shape) != (rows, k) or not out.is_contiguous():
        raise ValueError("out must be contiguous int32 [num_rows, k]")
    if logits.dtype == torch.float32 and not unsorted and index_table is None:
        rc = _lib.dsa_topk(logits.data_ptr(), stride, lengths.data_ptr(), rows, int(k), out.data_ptr(),
                           _stream_handle(stream))
    else:
        tptr, tstride = None, 0
        if index_table is not None:
            if (index_table.dtype != torch.int32 or index_table.dim() != 2 or not index_table.is_cuda
                    or index_table.size(0) != rows or (index_table.size(1) > 1 and index_table.stride(1) != 1)):
                raise ValueError("index_table must be a CUDA int32 [num_rows, >= max L] tensor with stride(1) == 1")
            tptr = index_table.data_ptr()
            tstride = int(index_table.stride(0)) if rows > 1 else max(int(index_table.size(1)), 1)
        rc = _lib.dsa_topk_ex(logits.data_ptr(), _DTYPES[logits.dtype], stride, lengths.data_ptr(), rows, int(k),
                              FLAG_UNSORTED if unsorted else 0, tptr, tstride, out.data_ptr(),
                              _stream_handle(stream))
    if rc != 0:
        raise DsaTopkError(rc)
    return out


def dsa_topk_host(logits: torch.Tensor, lengths: torch.Tensor, k: int, out: torch.Tensor,
                  d_logits: torch.Tensor, d_lengths: torch.Tensor, d_out: torch.Tensor,
                  stream=None) -> torch.Tensor:
    """Host-buffer variant: copies ``logits`` / ``lengths`` (CPU, ideally pinned)
    into the device staging tensors, runs the top-k and copies the result back
    into ``out`` (CPU int32 ``[rows, k]``), all on ``stream``. The caller
    synchronises the stream before reading ``out``."""
    rows, stride = _check_rows(logits, lengths, k)
    if logits.is_cuda or lengths.is_cuda or out.is_cuda:
        raise ValueError("host variant takes CPU tensors")
    if not logits.is_contiguous() and rows > 1 and logits.stride(0) != stride:
        raise ValueError("logits must be laid out at its row stride")
    for t, dt in ((d_logits, torch.float32), (d_lengths, torch.int32), (d_out, torch.int32)):
        if not t.is_cuda or t.dtype != dt:
            raise ValueError("device staging tensors must be CUDA tensors of the right dtype")
    if d_logits.numel() < rows * stride or d_lengths.numel() < rows or d_out.numel() < rows * k:
        raise ValueError("device staging tensors too small")
    rc = _lib.dsa_topk_host(logits.data_ptr(), stride, lengths.data_ptr(), rows, int(k), out.data_ptr(),
                            d_logits.data_ptr(), d_lengths.data_ptr(), d_out.data_ptr(), _stream_handle(stream))
    if rc != 0:
        raise DsaTopkError(rc)
    return out


def plan(num_rows: int, row_stride: int, k: int) -> Tuple[int, int]:
    """(cluster_size, grid) that dsa_topk picks on the current device."""
    cs, grid = _I32(0), _I32(0)
    rc = _lib.dsa_topk_plan(int(num_rows), int(row_stride), int(k), ctypes.byref(cs), ctypes.byref(grid))
    if rc != 0:
        raise DsaTopkError(rc)
    return cs.value, grid.value


def device_status(clear: bool = False) -> int:
    """Sticky device-side status bits (``STATUS_*``; ``STATUS_ERRORS`` are the
    error bits, ``STATUS_REREAD`` is informational). Syncs the device."""
    v = ctypes.c_uint32(0)
    rc = _lib.dsa_topk_device_status(ctypes.byref(v), 1 if clear else 0)
    if rc != 0:
        raise DsaTopkError(rc)
    return int(v.value)


def set_test_hooks(wait_limit_ns: int = 0, skip_stage: int = -1) -> None:
    """Test use only: the time limit of every device-side wait (0: default
    0.5 s) and a stage each CTA's producer leaves unissued (-1: none)."""
    rc = _lib.dsa_topk_set_test_hooks(int(wait_limit_ns), int(skip_stage))
    if rc != 0:
        raise DsaTopkError(rc)


__all__ = ["dsa_topk", "dsa_topk_host", "plan", "device_status", "set_test_hooks", "strerror", "version",
           "DTYPE_F32", "DTYPE_BF16", "DTYPE_F16", "FLAG_UNSORTED",
           "DsaTopkError", "MAX_K", "LIB_PATH", "lib", "STATUS_WAIT_TIMEOUT", "STATUS_SELECT_BROKEN",
           "STATUS_REREAD", "STATUS_ERRORS"]
