"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: hand-derived
cases, O(L^2) brute-force ranking, exhaustive special values, NumPy / PyTorch
stable sorts (the special case where the definition reduces to a textbook
stable argsort), closed forms, and invariants that must hold at any size.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import workloads
from tests.topk_checks import brute_force_row, check_all, check_row

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.txt")


def _parse_float(tok):
    return np.inf if tok == "pad" else float(tok)


def load_golden():
    cases, cur = [], {}
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.rstrip("\n")
        if line.startswith("#"):
            continue
        if not line.strip():
            if cur:
                cases.append(cur)
                cur = {}
            continue
        key, _, val = line.partition(":")
        cur[key.strip()] = val.strip()
    if cur:
        cases.append(cur)
    out = []
    for c in cases:
        logits = np.array([_parse_float(t) for t in c["logits"].split()], dtype=np.float32)
        expect = np.array([[int(t) for t in row.split()] for row in c["expect"].split("|")], dtype=np.int32)
        out.append(dict(
            name=c["case"], source=c["source"], k=int(c["k"]), row_stride=int(c["row_stride"]),
            lengths=np.array([int(t) for t in c["lengths"].split()], dtype=np.int32),
            logits=logits, expect=expect,
            wrong_stride=int(c["wrong_stride"]) if "wrong_stride" in c else None,
        ))
    return out


GOLDEN_CASES = load_golden()


@pytest.mark.parametrize("case", GOLDEN_CASES, ids=[c["name"] for c in GOLDEN_CASES])
def test_golden_hand_cases(oracle_mod, case):
    assert case["source"], "every golden case cites its source"
    got = oracle_mod.topk(case["logits"], case["lengths"], case["k"], row_stride=case["row_stride"])
    np.testing.assert_array_equal(got, case["expect"])
    if case["wrong_stride"] is not None:
        # the size(1)-for-stride(0) bug must change the answer on this fixture
        bad = oracle_mod.topk(case["logits"], case["lengths"], case["k"], row_stride=case["wrong_stride"])
        assert not np.array_equal(bad, case["expect"])


def test_brute_force_random_small(oracle_mod):
    rng = np.random.default_rng(123)
    for trial in range(300):
        L = int(rng.integers(0, 40))
        stride = L + int(rng.integers(0, 5)) if L else int(rng.integers(1, 5))
        # few distinct values so that ties are common; sprinkle specials
        pool = np.array([-2, -1, -0.0, 0.0, 0.5, 1, 3, np.inf, -np.inf, np.nan], dtype=np.float32)
        vals = pool[rng.integers(0, len(pool), size=L)]
        row = np.full(stride, np.inf, dtype=np.float32)
        row[:L] = vals
        for k in sorted({1, 2, max(1, L // 2), max(1, L), L + 3}):
            got = oracle_mod.topk(row[None, :], np.array([L], np.int32), k)[0]
            assert list(got) == brute_force_row(vals.tolist(), k), (trial, L, k)


def test_exhaustive_special_values(oracle_mod):
    """Every row of length <= 5 over {-inf, -1, -0.0, +0.0, 1, +inf, NaN}."""
    specials = [-np.inf, -1.0, -0.0, 0.0, 1.0, np.inf, np.nan]
    for L in range(0, 6):
        rows = list(itertools.product(specials, repeat=L)) if L else [()]
        stride = max(L, 1)
        a = np.full((len(rows), stride), np.inf, dtype=np.float32)
        for i, r in enumerate(rows):
            a[i, :L] = r
        lens = np.full(len(rows), L, dtype=np.int32)
        ref = [brute_force_row(list(r), 6) for r in rows]
        for k in range(1, 7):
            got = oracle_mod.topk(a, lens, k)
            exp = np.array([r[:k] for r in ref], dtype=np.int32).reshape(len(rows), k)
            np.testing.assert_array_equal(got, exp, err_msg="L=%d k=%d" % (L, k))


def test_matches_numpy_stable_argsort(oracle_mod):
    """Finite, NaN-free rows: the definition is numpy's stable argsort of -x."""
    rng = np.random.default_rng(7)
    for trial in range(40):
        L = int(rng.integers(1, 5000))
        k = int(rng.integers(1, 2049))
        levels = int(rng.integers(2, 50))
        vals = (rng.integers(0, levels, size=L) - levels // 2).astype(np.float32) * 0.25
        vals[rng.random(L) < 0.05] = -0.0
        row = np.concatenate([vals, np.full(7, np.inf, np.float32)])
        got = oracle_mod.topk(row[None, :], np.array([L], np.int32), k)[0]
        m = min(k, L)
        exp = np.argsort(-vals.astype(np.float64), kind="stable")[:m]
        np.testing.assert_array_equal(got[:m], exp)
        assert np.all(got[m:] == -1)


def test_matches_torch_stable_sort_and_topk_values(oracle_mod):
    g = torch.Generator().manual_seed(11)
    for trial in range(20):
        L = int(torch.randint(1, 20000, (1,), generator=g))
        k = int(torch.randint(1, 2049, (1,), generator=g))
        x = torch.randn(L, generator=g).to(torch.float8_e4m3fn).to(torch.float32)  # ties, +-0
        got = oracle_mod.topk(x.numpy()[None, :], np.array([L], np.int32), k)[0]
        m = min(k, L)
        exp = torch.sort(x, descending=True, stable=True).indices[:m].numpy()
        np.testing.assert_array_equal(got[:m], exp)
        # torch.topk's tie order is unspecified: compare the selected values only
        tv = torch.topk(x, m).values.numpy()
        np.testing.assert_array_equal(np.sort(x.numpy()[got[:m]]), np.sort(tv))


@pytest.mark.parametrize("L,k", [(1, 1), (7, 3), (1000, 512), (4096, 2048), (100, 2048)])
def test_closed_forms(oracle_mod, L, k):
    m = min(k, L)
    pad = np.full(5, np.inf, np.float32)
    lens = np.array([L], np.int32)
    expect_prefix = np.arange(m, dtype=np.int32)
    for row in (np.full(L, 0.75, np.float32),                       # all equal
                np.linspace(10, -10, L).astype(np.float32)):        # strictly decreasing
        got = oracle_mod.topk(np.concatenate([row, pad])[None], lens, k)[0]
        np.testing.assert_array_equal(got[:m], expect_prefix)
        assert np.all(got[m:] == -1)
    inc = np.arange(L, dtype=np.float32)                            # strictly increasing
    got = oracle_mod.topk(np.concatenate([inc, pad])[None], lens, k)[0]
    np.testing.assert_array_equal(got[:m], np.arange(L - 1, L - 1 - m, -1, dtype=np.int32))
    # L = 0: all -1
    got = oracle_mod.topk(np.concatenate([inc, pad])[None], np.array([0], np.int32), k)[0]
    assert np.all(got == -1)


def test_stride_and_poison_invariance(oracle_mod):
    """Same valid rows at other strides (incl. unaligned) and other padding."""
    wl = workloads.make_rows("decode", [0, 1, 2, 3, 17, 40])
    Lmax = int(wl.lengths.max())
    base = oracle_mod.topk(wl.logits, wl.lengths, wl.k)
    for stride in (Lmax, Lmax + 3, 2 * Lmax + 1):
        for poison in (np.inf, np.nan, -np.inf, 1e30):
            a = np.full((wl.num_rows, stride), poison, np.float32)
            for i in range(wl.num_rows):
                a[i, : wl.lengths[i]] = wl.logits[i, : wl.lengths[i]]
            np.testing.assert_array_equal(oracle_mod.topk(a, wl.lengths, wl.k), base)


@pytest.mark.parametrize("name,rows", [
    ("tiny", [0, 1, 2, 3]),
    ("decode", [0, 1, 2, 3, 5, 63]),
    ("ties", [0, 255]),
    ("prefill", [0, 4095]),
    ("cluster", [3]),
])
def test_invariants_on_workloads(oracle_mod, name, rows):
    wl = workloads.make_rows(name, rows)
    out = oracle_mod.topk(wl.logits, wl.lengths, wl.k)
    check_all(wl.logits, wl.lengths, wl.k, out)


def test_ties_workload_closed_form(oracle_mod):
    """16 levels: the top level 7.5 occurs >= 2048 times per row, so the
    answer is the first 2048 positions holding 7.5, ascending."""
    wl = workloads.make_rows("ties", [0, 1, 128, 255])
    out = oracle_mod.topk(wl.logits, wl.lengths, wl.k)
    for i in range(wl.num_rows):
        pos = np.nonzero(wl.logits[i, : wl.lengths[i]] == 7.5)[0]
        assert len(pos) >= wl.k
        np.testing.assert_array_equal(out[i], pos[: wl.k])


def test_cluster_workload_never_picks_neg_inf_tail(oracle_mod):
    wl = workloads.make_rows("cluster", [0])
    out = oracle_mod.topk(wl.logits, wl.lengths, wl.k)
    assert out.max() < workloads.CLUSTER_FINITE and out.min() >= 0


def test_multithreaded_equals_single_thread(oracle_mod):
    wl = workloads.make_rows("decode", range(0, 64, 3))
    a = oracle_mod.topk(wl.logits, wl.lengths, wl.k, threads=1)
    b = oracle_mod.topk(wl.logits, wl.lengths, wl.k, threads=8)
    np.testing.assert_array_equal(a, b)


def test_bad_arguments(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.topk(np.zeros((2, 4), np.float32), np.zeros(2, np.int32), 0)
