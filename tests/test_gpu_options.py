"""GPU parity of dsa_topk_ex's options against the oracle, on both launch
shapes (one CTA per row over many rows; a cluster per row over few long rows):

* bf16 / fp16 logits: the oracle runs on the same values widened to fp32
  (exact), so the expected indices are the fp32 definition applied to the
  16-bit values;
* the unsorted (set) output: per row, the same index set as the oracle, -1
  padding in place;
* the index table: the oracle's indices mapped through the table on the CPU,
  -1 passed through.

Every comparison is exact (integer outputs). Calls go through the C ABI.
"""
import zlib

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

SHAPES = {
    # name: (rows, width, k)  -- width is the row stride of the test buffer
    "rows": (300, 20000, 2048),
    "cluster": (4, 300000, 1024),
}


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_strided_b200 as m
    m.device_status(clear=True)
    return m


def _lengths(rng, rows, width, k):
    L = rng.integers(1, width + 1, size=rows).astype(np.int32)
    L[0], L[-1] = width, min(k // 2, width)  # a full row and a row shorter than k
    if rows > 2:
        L[1] = 0
    return L


def _values(rng, rows, width, special=False):
    x = rng.standard_normal((rows, width))
    x[1::3] = np.round(x[1::3] * 4) / 4  # ties
    if special:
        pool = np.array([np.nan, np.inf, -np.inf, 0.0, -0.0, 1.0], np.float64)
        mask = rng.random((rows, width)) < 0.02
        x[mask] = pool[rng.integers(0, len(pool), mask.sum())]
    return x


def _device_rows(t, base_offset):
    """The [rows, width] tensor `t` copied into a CUDA buffer starting
    `base_offset` elements in (odd offsets misalign the rows), as a view."""
    rows, width = t.shape
    buf = torch.full((base_offset + rows * width + 8,), float("inf"), dtype=t.dtype)
    buf[base_offset:base_offset + rows * width] = t.reshape(-1)
    d = buf.cuda()
    return d[base_offset:base_offset + rows * width].view(rows, width)


def _check_plan(dsa, shape, rows, width, k):
    cs = dsa.plan(rows, width, k)[0]
    assert (cs > 1) == (shape == "cluster"), (shape, cs)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape", list(SHAPES))
@pytest.mark.parametrize("base_offset", [0, 3])
def test_half_precision_logits(oracle_mod, dsa, dtype, shape, base_offset):
    rows, width, k = SHAPES[shape]
    rng = np.random.default_rng(zlib.crc32(("%s/%s/%d" % (dtype, shape, base_offset)).encode()))
    x16 = torch.from_numpy(_values(rng, rows, width, special=True)).to(dtype)  # round to nearest even
    L = _lengths(rng, rows, width, k)
    _check_plan(dsa, shape, rows, width, k)
    got = dsa.dsa_topk(_device_rows(x16, base_offset), torch.from_numpy(L).cuda(), k)
    exp = oracle_mod.topk(x16.float().numpy(), L, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got.cpu().numpy(), exp)
    assert dsa.device_status() & dsa.STATUS_ERRORS == 0


@pytest.mark.parametrize("shape", list(SHAPES))
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_unsorted_output_is_the_same_set(oracle_mod, dsa, shape, dtype):
    rows, width, k = SHAPES[shape]
    rng = np.random.default_rng(7 + len(shape))
    xt = torch.from_numpy(_values(rng, rows, width)).to(dtype)
    L = _lengths(rng, rows, width, k)
    _check_plan(dsa, shape, rows, width, k)
    got = dsa.dsa_topk(xt.cuda(), torch.from_numpy(L).cuda(), k, unsorted=True).cpu().numpy()
    exp = oracle_mod.topk(xt.float().numpy(), L, k)
    for r in range(rows):
        m = min(k, int(L[r]))
        np.testing.assert_array_equal(np.sort(got[r, :m]), np.sort(exp[r, :m]), err_msg="row %d" % r)
        assert np.all(got[r, m:] == -1)


@pytest.mark.parametrize("shape", list(SHAPES))
def test_index_table_maps_every_index(oracle_mod, dsa, shape):
    rows, width, k = SHAPES[shape]
    rng = np.random.default_rng(11 + len(shape))
    x = _values(rng, rows, width).astype(np.float32)
    L = _lengths(rng, rows, width, k)
    tstride = width + 5
    table = rng.integers(-2 ** 31, 2 ** 31 - 1, size=(rows, tstride), dtype=np.int64).astype(np.int32)
    d_table = torch.from_numpy(table).cuda()[:, :width]  # a strided view: row stride tstride
    _check_plan(dsa, shape, rows, width, k)
    got = dsa.dsa_topk(torch.from_numpy(x).cuda(), torch.from_numpy(L).cuda(), k, index_table=d_table)
    idx = oracle_mod.topk(x, L, k)
    exp = np.where(idx >= 0, np.take_along_axis(table, np.maximum(idx, 0), axis=1), -1)
    np.testing.assert_array_equal(got.cpu().numpy(), exp)


def test_all_options_together(oracle_mod, dsa):
    """fp16 logits, unsorted output and an index table in one cluster call."""
    rows, width, k = SHAPES["cluster"]
    rng = np.random.default_rng(99)
    x16 = torch.from_numpy(_values(rng, rows, width)).to(torch.float16)
    L = _lengths(rng, rows, width, k)
    table = rng.integers(0, 1 << 30, size=(rows, width), dtype=np.int64).astype(np.int32)
    got = dsa.dsa_topk(x16.cuda(), torch.from_numpy(L).cuda(), k, unsorted=True,
                       index_table=torch.from_numpy(table).cuda()).cpu().numpy()
    idx = oracle_mod.topk(x16.float().numpy(), L, k)
    exp = np.where(idx >= 0, np.take_along_axis(table, np.maximum(idx, 0), axis=1), -1)
    for r in range(rows):
        m = min(k, int(L[r]))
        np.testing.assert_array_equal(np.sort(got[r, :m]), np.sort(exp[r, :m]))
        assert np.all(got[r, m:] == -1)


def test_bf16_prefill_rows(oracle_mod, dsa):
    """Prefill-shaped rows (L_i = 126977 + i, stride 131072, k = 2048) in bf16,
    296 rows so that every CTA carries estimates between its rows."""
    import workloads
    wl = workloads.make_rows("prefill", range(296))
    x16 = torch.from_numpy(wl.logits).to(torch.bfloat16)
    got = dsa.dsa_topk(x16.cuda(), torch.from_numpy(wl.lengths).cuda(), wl.k)
    exp = oracle_mod.topk(x16.float().numpy(), wl.lengths, wl.k)
    np.testing.assert_array_equal(got.cpu().numpy(), exp)
