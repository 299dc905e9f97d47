"""The seeded input generators: shapes, recipes, determinism (no GPU)."""
import numpy as np
import pytest
import torch

import workloads


def test_e4m3_rounding_matches_torch_float8():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000) * s for s in (1e-3, 0.1, 1, 30)])
    x = np.concatenate([x, [0.0, -0.0, 1.0625, 1.1875, -2.5625, 2 ** -9 * 1.5, 2 ** -10, 447.9, 463.9]])
    # above 464 torch's conversion overflows to NaN while round_to_e4m3 saturates;
    # the N(0,1) recipe never gets there
    x = x[np.abs(x) < 464]
    ours = workloads.round_to_e4m3(x).astype(np.float32)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    # compare bit patterns so -0.0 vs +0.0 counts
    np.testing.assert_array_equal(ours.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("name", workloads.CONFIG_NAMES)
def test_lengths_and_shapes(name):
    s = workloads.spec(name)
    L = workloads.lengths_of(name)
    assert L.dtype == np.int32 and L.shape == (s.num_rows,)
    assert L.min() >= 1 and L.max() <= s.row_stride
    if name == "decode":
        assert list(L[:4]) == [1, 1000, 2048, 65536]
    if name == "prefill":
        assert L[0] == 126977 and L[-1] == 131072
    if name == "cluster":
        assert s.row_stride % 256 == 0 and s.row_stride > 900000


@pytest.mark.parametrize("name", ["tiny", "decode", "ties"])
def test_rows_regenerate_bit_exactly(name):
    rows = [0, 2, 3]
    a = workloads.make_rows(name, rows)
    b = workloads.make_rows(name, rows, row_stride=workloads.spec(name).row_stride + 5)
    for i in range(len(rows)):
        L = a.lengths[i]
        np.testing.assert_array_equal(a.logits[i, :L].view(np.uint32), b.logits[i, :L].view(np.uint32))
        assert np.all(np.isposinf(a.logits[i, L:]))


def test_value_recipes():
    d = workloads.make_rows("decode", [3])
    v = d.logits[0, : d.lengths[0]].astype(np.float64)
    np.testing.assert_array_equal(workloads.round_to_e4m3(v), v)  # already on the fp8 grid
    assert np.any(np.signbit(v) & (v == 0))  # -0.0 present
    t = workloads.make_rows("ties", [7])
    assert set(np.unique(t.logits[0, : t.lengths[0]])) <= set(workloads.TIES_LEVELS.tolist())
    c = workloads.make_rows("cluster", [1])
    row = c.logits[0]
    assert np.all(np.isneginf(row[810000:900000])) and np.all(np.isfinite(row[:810000]))
    p = workloads.make_rows("prefill", [0])
    L = p.lengths[0]
    # far keys carry the +0.5*log1p(d) bias, d = (L-1) - j
    d = (L - 1) - np.arange(L)
    resid = p.logits[0, :L].astype(np.float64) - 0.5 * np.log1p(d)
    assert abs(resid.mean()) < 0.02 and abs(resid.std() - 1.0) < 0.02


def test_valid_bytes():
    assert workloads.valid_bytes(workloads.lengths_of("prefill")) == 2113937408
    assert workloads.valid_bytes(workloads.lengths_of("ties")) == 134217728
    assert workloads.valid_bytes(workloads.lengths_of("cluster")) == 14400000
