"""The oracle's pins must catch plausible mistakes.

Each mutant below is the oracle source with one plausible error planted (on
the CPU, in a temporary copy). The test compiles it and requires that at least
one pin from test_oracle.py-style checks rejects it. A pin set that passes a
mutant would not be pinning the part the mutant breaks.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

import workloads
from tests.test_oracle import GOLDEN_CASES
from tests.topk_checks import brute_force_row

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "dsa_topk_oracle.cpp")

MUTANTS = {
    # P1's bug: the row base taken from the valid width instead of the row stride
    "stride_is_width": ("one_row(logits + r * row_stride,", "one_row(logits + r * static_cast<int64_t>(lengths[0]),"),
    # ties resolved by highest index instead of lowest
    "ties_high_index_first": ("std::stable_sort(order.begin(), order.end(),",
                              "std::reverse(order.begin(), order.end()); std::stable_sort(order.begin(), order.end(),"),
    # NaN ranked at the bottom instead of above +inf
    "nan_lowest": ("if (na || nb) return na && !nb;", "if (na || nb) return nb && !na;"),
    # padding filled with 0 instead of -1
    "pad_zero": ("? order[static_cast<size_t>(t)] : -1;", "? order[static_cast<size_t>(t)] : 0;"),
    # ascending instead of descending
    "ascending": ("return a > b;  //", "return a < b;  //"),
    # -0.0 ranked below +0.0
    "signed_zero_split": ("return a > b;  //", "return a > b || (a == b && !std::signbit(a) && std::signbit(b));  //"),
    # lengths not clamped to the stride (reads the neighbouring row's data)
    "no_upper_clamp": ("if (L > row_stride) L = row_stride;", ""),
    # k clipped one short
    "m_off_by_one": ("const int64_t m = std::min<int64_t>(k, L);", "const int64_t m = std::min<int64_t>(k, L) - (L > 1 ? 1 : 0);"),
}


def _build(tmpdir, name, old, new):
    src = open(SRC).read()
    assert old in src, "mutation anchor missing for %s" % name
    path_c = os.path.join(tmpdir, name + ".cpp")
    path_so = os.path.join(tmpdir, name + ".so")
    open(path_c, "w").write(src.replace(old, new, 1))
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-pthread", path_c, "-o", path_so])
    lib = ctypes.CDLL(path_so)
    lib.oracle_dsa_topk.restype = ctypes.c_int
    lib.oracle_dsa_topk.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                    ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32]

    def topk(logits, lengths, k, row_stride):
        a = np.ascontiguousarray(logits, np.float32)
        L = np.ascontiguousarray(lengths, np.int32)
        # slack after the buffer so an unclamped mutant reads memory it owns
        buf = np.concatenate([a.ravel(), np.full(4 * row_stride + 64, np.inf, np.float32)])
        out = np.empty((len(L), k), np.int32)
        lib.oracle_dsa_topk(buf.ctypes.data, row_stride, L.ctypes.data, len(L), k, out.ctypes.data, 1)
        return out
    return topk


def _pins_fail(topk) -> list:
    failed = []
    for c in GOLDEN_CASES:
        got = topk(c["logits"], c["lengths"], c["k"], c["row_stride"])
        if not np.array_equal(got, c["expect"]):
            failed.append("golden:" + c["name"])
    rng = np.random.default_rng(5)
    pool = np.array([-2, -1, -0.0, 0.0, 1, 3, np.inf, -np.inf, np.nan], np.float32)
    for t in range(60):
        L = int(rng.integers(1, 12))
        vals = pool[rng.integers(0, len(pool), L)]
        for k in (1, L, L + 2):
            if list(topk(vals[None], np.array([L], np.int32), k, L)[0]) != brute_force_row(vals.tolist(), k):
                failed.append("brute_force")
                break
    wl = workloads.make_rows("decode", [1, 2, 5])
    a = topk(wl.logits, wl.lengths, wl.k, wl.row_stride)
    b = topk(np.ascontiguousarray(wl.logits[:, : int(wl.lengths.max()) + 3]), wl.lengths, wl.k, int(wl.lengths.max()) + 3)
    if not np.array_equal(a, b):
        failed.append("stride_invariance")
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with tempfile.TemporaryDirectory() as d:
        topk = _build(d, name, old, new)
        failed = _pins_fail(topk)
    assert failed, "mutant %s passed every pin" % name


def test_unmutated_source_passes_same_pins():
    with tempfile.TemporaryDirectory() as d:
        topk = _build(d, "identity", "extern \"C\" {", "extern \"C\" {")
        assert _pins_fail(topk) == []
