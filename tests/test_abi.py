"""The C-ABI library loads and exports exactly what include/dsa_topk.h declares.

No compute calls here: argument checks return before the library touches the
CUDA runtime, so they run without a GPU.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa_topk.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(dsa_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def pkg():
    import __graft_entry__

    __graft_entry__.build()
    import sparse_attention_indexer_strided_b200 as m
    return m


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("dsa_topk", "dsa_topk_ex", "dsa_topk_host", "dsa_topk_plan", "dsa_topk_device_status",
              "dsa_topk_set_test_hooks", "dsa_topk_strerror", "dsa_topk_version"):
        assert n in names


def test_library_exports_every_declared_symbol(pkg):
    lib = ctypes.CDLL(pkg.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", pkg.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted(l.split()[-1] for l in out.splitlines() if l.split() and l.split()[-1].startswith("dsa_"))
    assert exported == declared_functions(), "exports must match the header exactly"
    others = [l.split()[-1] for l in out.splitlines() if l.split() and not l.split()[-1].startswith(("dsa_", "_"))]
    assert others == [], "unexpected exported symbols: %s" % others[:5]


def test_strerror_and_version(pkg):
    assert pkg.version() >= 100
    assert pkg.strerror(0) == "success"
    for code in range(-11, 0):
        assert pkg.strerror(code) and pkg.strerror(code) != pkg.strerror(1)


@pytest.mark.parametrize("args,code", [
    # (logits, row_stride, lengths, num_rows, k, out)
    ((8, 16, 8, 2, 0, 8), -2),      # k = 0
    ((8, 16, 8, 2, 2049, 8), -2),   # k too large
    ((8, 0, 8, 2, 4, 8), -3),       # stride 0
    ((8, 16, 8, -1, 4, 8), -4),     # negative rows
    ((8, 2 ** 62, 8, 4, 4, 8), -5), # rows*stride overflows
    ((0, 16, 8, 2, 4, 8), -1),      # null logits
    ((8, 16, 0, 2, 4, 8), -1),      # null lengths
    ((8, 16, 8, 2, 4, 0), -1),      # null out
    ((9, 16, 8, 2, 4, 8), -6),      # misaligned logits
    ((8, 16, 8, 2, 4, 10), -6),     # misaligned out
])
def test_argument_errors_return_codes(pkg, args, code):
    lo, stride, le, rows, k, out = args
    rc = pkg.lib.dsa_topk(lo or None, stride, le or None, rows, k, out or None, None)
    assert rc == code


def test_zero_rows_is_a_no_op(pkg):
    assert pkg.lib.dsa_topk(None, 16, None, 0, 4, None, None) == 0


def test_plan_rejects_bad_sizes(pkg):
    assert pkg.lib.dsa_topk_plan(4, 16, 0, None, None) == -2
    assert pkg.lib.dsa_topk_plan(4, 0, 8, None, None) == -3
    assert pkg.lib.dsa_topk_plan(-4, 16, 8, None, None) == -4


@pytest.mark.parametrize("args,code", [
    # (logits, dtype, row_stride, lengths, num_rows, k, flags, table, table_stride, out)
    ((8, 3, 16, 8, 2, 4, 0, 0, 0, 8), -10),    # unknown dtype
    ((8, 0, 16, 8, 2, 4, 2, 0, 0, 8), -11),    # unknown flag bit
    ((8, 0, 16, 8, 2, 4, 0, 8, 0, 8), -3),     # table without a positive stride
    ((10, 1, 16, 8, 2, 4, 0, 0, 0, 8), 0),     # bf16 needs 2-byte alignment only: reaches the device check
    ((9, 1, 16, 8, 2, 4, 0, 0, 0, 8), -6),     # misaligned bf16 logits
    ((8, 0, 16, 8, 2, 4, 0, 10, 3, 8), -6),    # misaligned table
    ((8, 2, 16, 8, 0, 4, 1, 0, 0, 8), 0),      # zero rows: no-op
])
def test_ex_argument_errors(pkg, args, code):
    lo, dt, stride, le, rows, k, flags, tab, ts, out = args
    rc = pkg.lib.dsa_topk_ex(lo or None, dt, stride, le or None, rows, k, flags, tab or None, ts, out or None, None)
    if code == 0 and rows:
        assert rc in (0, -7)  # -7: no sm_100a device here
    else:
        assert rc == code
