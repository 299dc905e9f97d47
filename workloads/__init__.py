"""Seeded synthetic inputs for the strided indexer top-k.

This module only *draws* inputs. It holds none of the top-k arithmetic, so the
CPU oracle and the CUDA path can both consume it without sharing any logic.

Each workload stands in for the indexer logits that a DeepSeek-V4 serving
stack hands to its top-k kernel (vLLM PR #42169 page, "功能与动机": the
DeepGEMM logits are padded to a multiple of 256 along the context dimension
and then sliced, so rows are addressed with a row stride larger than the valid
length). The model itself, its weights and the GPQA / gsm8k evaluation sets
the pages use are not available, so values come from the recipes below.

Recipes (all padding ``[L_i, row_stride)`` is filled with ``+inf`` poison, so a
kernel that reads past ``L_i`` or uses the wrong stride picks a poisoned entry):

* ``tiny``    4 rows, stride 4096, L=4000, N(0,1), seed 0, k=512.
* ``decode``  64 rows, stride 65536, L_i ~ U{1..65536} (seed 1), rows 0-3 forced
  to L = 1, 1000, 2048, 65536; N(0,1) rounded to the fp8 e4m3 grid
  (round-to-nearest-even) and stored as fp32 (this creates ties and -0.0);
  k=2048.
* ``cluster`` 4 rows, stride 900096, L=900000, N(0,1) seed 2, the last 10% of
  each row set to -inf, k=1024.
* ``prefill`` 4096 rows (the last 4096 query positions of a 131072-token
  context), stride 131072, L_i = 126977 + i, value = N(0,1) (seed 3) +
  0.5*log1p(d) with d = (L_i - 1) - j the distance to the query, formed in
  fp64 and rounded to fp32, k=2048.
* ``ties``    256 rows, stride 131328, L=131072, values drawn uniformly from
  the 16 levels {-7.5, -6.5, ..., 7.5} (seed 4), k=2048.

Every row has its own random stream, ``numpy.random.default_rng([seed, 1,
row])``; per-row lengths come from ``default_rng([seed, 0])``. Any subset of
rows can therefore be regenerated on its own, bit for bit, which is how the
full-size parity tests feed sampled rows to the oracle.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import hashlib
import os
from typing import Dict, Iterable, List, Optional

import numpy as np

__all__ = [
    "Workload",
    "CONFIG_NAMES",
    "spec",
    "make",
    "make_rows",
    "round_to_e4m3",
    "valid_bytes",
    "sha256",
]

CONFIG_NAMES = ("tiny", "decode", "cluster", "prefill", "ties")


@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    num_rows: int
    row_stride: int
    k: int
    seed: int


_SPECS: Dict[str, Spec] = {
    "tiny": Spec("tiny", 4, 4096, 512, 0),
    "decode": Spec("decode", 64, 65536, 2048, 1),
    "cluster": Spec("cluster", 4, 900096, 1024, 2),
    "prefill": Spec("prefill", 4096, 131072, 2048, 3),
    "ties": Spec("ties", 256, 131328, 2048, 4),
}

TIES_LEVELS = np.arange(16, dtype=np.float64) - 7.5  # -7.5 ... 7.5
CLUSTER_FINITE = 810000  # cluster rows: [810000, 900000) is -inf


@dataclasses.dataclass
class Workload:
    name: str
    logits: np.ndarray  # float32 [num_rows, row_stride], padding = +inf
    lengths: np.ndarray  # int32 [num_rows]
    k: int

    @property
    def num_rows(self) -> int:
        return int(self.logits.shape[0])

    @property
    def row_stride(self) -> int:
        return int(self.logits.shape[1])


def spec(name: str) -> Spec:
    return _SPECS[name]


def round_to_e4m3(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest fp8 e4m3 (fn) value, ties to even.

    e4m3: 3 stored mantissa bits, exponent bias 7, smallest normal 2**-6,
    subnormal spacing 2**-9, largest finite 448 (saturated here). Scaling by
    powers of two is exact in fp64, so ``rint`` (half-to-even) on the scaled
    value is the round-to-nearest-even of the format.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)  # a = m * 2**ex, m in [0.5, 1)  ->  floor(log2 a) = ex - 1
    e = np.maximum(ex.astype(np.int64) - 1, -6)
    q = np.ldexp(1.0, e - 3)
    r = np.minimum(np.rint(a / q) * q, 448.0)
    return np.copysign(r, x)


def _lengths(s: Spec) -> np.ndarray:
    n = s.num_rows
    if s.name == "tiny":
        return np.full(n, 4000, dtype=np.int32)
    if s.name == "decode":
        rng = np.random.default_rng([s.seed, 0])
        L = rng.integers(1, 65536, size=n, endpoint=True).astype(np.int32)
        L[:4] = (1, 1000, 2048, 65536)
        return L
    if s.name == "cluster":
        return np.full(n, 900000, dtype=np.int32)
    if s.name == "prefill":
        return (126977 + np.arange(n)).astype(np.int32)
    if s.name == "ties":
        return np.full(n, 131072, dtype=np.int32)
    raise KeyError(s.name)


_LOG1P_CACHE: Dict[int, np.ndarray] = {}


def _half_log1p(n: int) -> np.ndarray:
    """0.5*log1p(d) for d = 0 .. n-1 (prefixes of one cached table)."""
    t = _LOG1P_CACHE.get(0)
    if t is None or len(t) < n:
        t = 0.5 * np.log1p(np.arange(max(n, 131072), dtype=np.float64))
        _LOG1P_CACHE[0] = t
    return t[:n]


def _row_values(s: Spec, row: int, L: int) -> np.ndarray:
    """The L valid fp32 values of one row (no padding)."""
    rng = np.random.default_rng([s.seed, 1, row])
    if s.name in ("tiny", "cluster"):
        v = rng.standard_normal(L, dtype=np.float32)
        if s.name == "cluster":
            v[CLUSTER_FINITE:] = -np.inf
        return v
    if s.name == "decode":
        return round_to_e4m3(rng.standard_normal(L)).astype(np.float32)
    if s.name == "prefill":
        n = rng.standard_normal(L)
        d_term = _half_log1p(L)[::-1]  # entry j holds 0.5*log1p(L-1-j)
        return (n + d_term).astype(np.float32)
    if s.name == "ties":
        return TIES_LEVELS[rng.integers(0, 16, size=L)].astype(np.float32)
    raise KeyError(s.name)


def make_rows(name: str, rows: Iterable[int], row_stride: Optional[int] = None,
              threads: int = 0) -> Workload:
    """Regenerate only ``rows`` of a workload, laid out at ``row_stride``.

    ``row_stride`` defaults to the workload's own stride; any stride >= the
    longest selected row gives the same valid values (padding is +inf).
    Rows have independent streams, so they are filled by a thread pool
    (``threads`` <= 0: one per CPU); the result does not depend on it.
    """
    s = _SPECS[name]
    rows = [int(r) for r in rows]
    L_all = _lengths(s)
    L = L_all[rows].astype(np.int32)
    stride = s.row_stride if row_stride is None else int(row_stride)
    if len(rows) and stride < int(L.max()):
        raise ValueError("row_stride shorter than a selected row")
    out = np.empty((len(rows), stride), dtype=np.float32)
    if s.name == "prefill":
        _half_log1p(int(L.max()) if len(rows) else 1)  # fill the shared table once

    def fill(i: int) -> None:
        out[i, : L[i]] = _row_values(s, rows[i], int(L[i]))
        out[i, L[i]:] = np.inf

    nt = threads if threads > 0 else (os.cpu_count() or 1)
    if nt <= 1 or len(rows) < 8:
        for i in range(len(rows)):
            fill(i)
    else:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(nt, 32)) as ex:
            list(ex.map(fill, range(len(rows))))
    return Workload(name=name, logits=out, lengths=L, k=s.k)


def make(name: str) -> Workload:
    """The full workload, exactly as specified (all rows, native stride)."""
    s = _SPECS[name]
    return make_rows(name, range(s.num_rows))


def valid_bytes(lengths: np.ndarray) -> int:
    """Algorithmic bytes of one call: every valid fp32 logit read once."""
    return 4 * int(np.asarray(lengths, dtype=np.int64).sum())


def sha256(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def lengths_of(name: str) -> np.ndarray:
    return _lengths(_SPECS[name])
