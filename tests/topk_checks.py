"""Checks on top-k outputs that do not use the oracle.

Used to pin the oracle and, on the GPU, as an extra net beside parity. The
order here is written independently of the oracle's comparator: a value maps
to the pair ``(is_nan, value)`` compared lexicographically (NaN above +inf,
all NaNs equal; -0.0 == +0.0 because float comparison treats them as equal).
"""
from __future__ import annotations

import math
from typing import Sequence

import numpy as np


def order_key(x: float):
    x = float(x)
    return (1, 0.0) if math.isnan(x) else (0, x)


def brute_force_row(vals: Sequence[float], k: int) -> list:
    """O(L^2) ranking: rank(j) = #{i: v_i > v_j} + #{i < j: v_i == v_j}."""
    keys = [order_key(v) for v in vals]
    L = len(keys)
    m = min(k, L)
    out = [-1] * k
    for j in range(L):
        r = 0
        for i in range(L):
            if keys[i] > keys[j] or (i < j and keys[i] == keys[j]):
                r += 1
        if r < m:
            out[r] = j
    return out


def _pairs(v: np.ndarray):
    """(nan_flag int8, value float64) with NaN values zeroed and -0.0 -> +0.0."""
    v = np.asarray(v, dtype=np.float64)
    isn = np.isnan(v)
    val = np.where(isn, 0.0, v) + 0.0  # adding +0.0 turns -0.0 into +0.0
    return isn.astype(np.int8), val


def check_row(vals: np.ndarray, L: int, k: int, out_row: np.ndarray) -> None:
    """Assert every invariant the definition implies for one row.

    ``vals`` holds at least the valid prefix (length L); ``out_row`` is the
    row's k output indices.
    """
    vals = np.asarray(vals)[:L]
    out_row = np.asarray(out_row)
    m = min(k, L)
    assert out_row.shape == (k,)
    assert np.all(out_row[m:] == -1), "padding must be -1 past min(k, L)"
    sel = out_row[:m].astype(np.int64)
    assert np.all((sel >= 0) & (sel < L)), "indices outside [0, L)"
    assert len(np.unique(sel)) == m, "repeated index"
    if m == 0:
        return
    fl, val = _pairs(vals)
    sf, sv = fl[sel], val[sel]
    # non-increasing along t; equal neighbours ascend in index
    dec = (sf[:-1] > sf[1:]) | ((sf[:-1] == sf[1:]) & (sv[:-1] > sv[1:]))
    eq = (sf[:-1] == sf[1:]) & (sv[:-1] == sv[1:])
    assert np.all(dec | eq), "output not ordered by value descending"
    assert np.all(sel[:-1][eq] < sel[1:][eq]), "ties not in ascending index order"
    if m < L:
        mask = np.ones(L, dtype=bool)
        mask[sel] = False
        uf, uv = fl[mask], val[mask]
        lf, lv = sf[-1], sv[-1]
        # min(selected) >= max(unselected)
        if uf.max() == 1:
            assert lf == 1, "an unselected NaN outranks a selected number"
        else:
            assert lf == 1 or lv >= uv.max(), "min(selected) < max(unselected)"
        # unselected entries tied with the last selected value lie after every
        # selected entry of that value
        tie_u = (uf == lf) & (uv == lv)
        if tie_u.any():
            unsel_idx = np.nonzero(mask)[0][tie_u]
            sel_tie = sel[(sf == lf) & (sv == lv)]
            assert unsel_idx.min() > sel_tie.max(), "tie broken against the lower index"


def check_all(logits2d: np.ndarray, lengths: np.ndarray, k: int, out: np.ndarray) -> None:
    """check_row over every row; out[i] belongs to logits2d[i] / lengths[i]."""
    stride = logits2d.shape[1]
    for i in range(logits2d.shape[0]):
        L = int(min(max(int(lengths[i]), 0), stride))
        check_row(logits2d[i], L, k, out[i])
