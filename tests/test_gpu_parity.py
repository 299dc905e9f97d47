"""GPU parity: the CUDA path against the CPU oracle, index for index.

All inputs are seeded. Every comparison is exact (integer outputs). Calls go
through the C ABI (ctypes) with torch used only for device memory and streams.
"""
import numpy as np
import pytest
import torch

import workloads
from tests.topk_checks import check_all

pytestmark = pytest.mark.gpu

CANARY = -123456789


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_strided_b200 as m
    m.device_status(clear=True)
    return m


def run_gpu(dsa, logits2d, lengths, k, base_offset=0, stride=None):
    """Lay rows out on the device at `stride` (default: the array's own),
    starting `base_offset` floats into the buffer, call dsa_topk through the
    C ABI and return the [rows, k] result. Guard words around the output must
    survive."""
    logits2d = np.asarray(logits2d, np.float32)
    rows, width = logits2d.shape
    stride = width if stride is None else stride
    assert stride >= width or rows <= 1
    buf = torch.full((base_offset + max(rows, 1) * stride + 8,), float("inf"), dtype=torch.float32)
    view = buf[base_offset: base_offset + rows * stride].view(rows, stride) if rows else None
    if rows:
        view[:, :width] = torch.from_numpy(logits2d)
    d_buf = buf.cuda()
    d_len = torch.from_numpy(np.asarray(lengths, np.int32).copy()).cuda()
    d_out = torch.full((rows * k + 64,), CANARY, dtype=torch.int32, device="cuda")
    out_ptr = d_out.data_ptr() + 32 * 4
    rc = dsa.lib.dsa_topk(d_buf.data_ptr() + 4 * base_offset, stride, d_len.data_ptr(), rows, k, out_ptr,
                          torch.cuda.current_stream().cuda_stream)
    assert rc == 0, dsa.strerror(rc)
    torch.cuda.synchronize()
    o = d_out.cpu().numpy()
    assert np.all(o[:32] == CANARY) and np.all(o[32 + rows * k:] == CANARY), "output guard words overwritten"
    return o[32:32 + rows * k].reshape(rows, k)


def assert_parity(oracle_mod, dsa, logits2d, lengths, k, **kw):
    got = run_gpu(dsa, logits2d, lengths, k, **kw)
    exp = oracle_mod.topk(logits2d, lengths, k)
    if not np.array_equal(got, exp):
        bad = np.nonzero(np.any(got != exp, axis=1))[0]
        r = bad[0]
        j = np.nonzero(got[r] != exp[r])[0][0]
        raise AssertionError("mismatch in %d rows; first row %d (L=%d) at t=%d: gpu %s oracle %s" % (
            len(bad), r, lengths[r], j, got[r, j:j + 6], exp[r, j:j + 6]))
    return got


# ------------------------------------------------------------ the 5 workloads
@pytest.mark.parametrize("name", ["tiny", "decode", "cluster", "ties"])
def test_workload_full_parity(oracle_mod, dsa, name):
    wl = workloads.make(name)
    got = assert_parity(oracle_mod, dsa, wl.logits, wl.lengths, wl.k)
    check_all(wl.logits, wl.lengths, wl.k, got)


def test_prefill_full_size_every_row(oracle_mod, dsa):
    """The full prefill batch (4096 rows, the benchmark's launch) against the
    oracle, every row index for index."""
    wl = workloads.make("prefill")
    assert dsa.plan(wl.num_rows, wl.row_stride, wl.k)[0] == 1
    got = run_gpu(dsa, wl.logits, wl.lengths, wl.k)
    exp = oracle_mod.topk(wl.logits, wl.lengths, wl.k)
    bad = np.nonzero(np.any(got != exp, axis=1))[0]
    assert len(bad) == 0, "%d of 4096 prefill rows differ, first %d" % (len(bad), bad[0])
    assert dsa.device_status() & dsa.STATUS_ERRORS == 0


def test_plan_choices(dsa):
    """Dispatch picks the cluster path for few long rows only."""
    assert dsa.plan(4096, 131072, 2048)[0] == 1
    assert dsa.plan(256, 131328, 2048)[0] == 1
    assert dsa.plan(4, 4096, 512)[0] == 1
    assert dsa.plan(4, 900096, 1024)[0] > 1
    assert dsa.plan(64, 65536, 2048)[0] == 1  # decode rows: one CTA each
    assert dsa.plan(64, 300000, 2048)[0] > 1  # many long rows: clusters


# ------------------------------------------------------------------ k sweep
LEN_MIX = [0, 1, 2, 30, 31, 32, 254, 255, 511, 512, 513, 1023, 1024, 1025, 2047, 2048, 2049,
           4095, 4096, 4097, 8191, 8192, 8193, 10239, 10240, 10241, 12288, 20000, 33333]


@pytest.mark.parametrize("k", [1, 31, 255, 512, 1023, 1024, 2047, 2048])
def test_k_sweep_many_rows(oracle_mod, dsa, k):
    rng = np.random.default_rng(1000 + k)
    stride = max(LEN_MIX) + 3
    rows = len(LEN_MIX) * 6  # >= SM count: one CTA per row
    L = np.array((LEN_MIX * 6)[:rows], np.int32)
    x = rng.standard_normal((rows, stride)).astype(np.float32)
    x[1::3] = np.round(x[1::3] * 4) / 4  # coarse grid: ties at the threshold
    assert_parity(oracle_mod, dsa, x, L, k)


@pytest.mark.parametrize("k", [1, 255, 1024, 2048])
def test_k_sweep_cluster_path(oracle_mod, dsa, k):
    rng = np.random.default_rng(2000 + k)
    stride = 300000
    L = np.array([300000, 123457, 20000, 2047, 0, 299999], np.int32)
    x = rng.standard_normal((len(L), stride)).astype(np.float32)
    x[2] = np.round(x[2] * 2) / 2
    assert dsa.plan(len(L), stride, k)[0] > 1
    assert_parity(oracle_mod, dsa, x, L, k)


def test_cluster_path_many_rows(oracle_mod, dsa):
    """32 rows and more take clusters only when rows are long: 40 long rows
    of mixed lengths, every fifth on a coarse grid."""
    rng = np.random.default_rng(2500)
    stride = 270000
    L = rng.integers(0, stride + 1, size=40).astype(np.int32)
    L[:4] = [stride, 0, 2048, 20000]
    x = rng.standard_normal((len(L), stride)).astype(np.float32)
    x[::5] = np.round(x[::5] * 8) / 8
    assert dsa.plan(len(L), stride, 2048)[0] > 1
    assert_parity(oracle_mod, dsa, x, L, 2048)


@pytest.mark.parametrize("seed", range(16))
def test_rows_random_shapes(oracle_mod, dsa, seed):
    """Seeded random many-row launches: 32-500 rows (one or two per CTA, where
    first rows sample 2048 values, or more, where they sample 4096 and later
    rows carry thresholds), strides 1000-200000 (the one-stage instance
    included), lengths from 0 to the stride, k from 1 to 2048, fp32 or bf16,
    and per row one of several value patterns."""
    rng = np.random.default_rng(3900 + seed)
    rows = int(rng.integers(32, 501))
    stride = int(rng.integers(1000, 200001))
    k = (2048, 512, 7, 2048, 1024, 1, 2048, 100)[seed % 8]
    L = rng.integers(0, stride + 1, size=rows).astype(np.int32)
    L[rng.random(rows) < 0.3] = stride
    x = rng.standard_normal((rows, stride)).astype(np.float32)
    kinds = rng.integers(0, 6, size=rows)
    x[kinds == 1] = np.round(x[kinds == 1] * 4) / 4
    x[kinds == 2] = rng.integers(0, 4, (int((kinds == 2).sum()), stride)).astype(np.float32)
    x[kinds == 3] = np.where(rng.random((int((kinds == 3).sum()), stride)) < 0.01, x[kinds == 3], -np.inf)
    x[kinds == 4] = np.sort(x[kinds == 4], axis=1)
    x[kinds == 5] = x[kinds == 5] - 2.0 * np.arange(int((kinds == 5).sum()))[:, None]
    t = torch.from_numpy(x)
    if seed % 2:
        t = t.to(torch.bfloat16)
    if dsa.plan(rows, stride, k)[0] != 1:
        pytest.skip("this shape takes clusters on this GPU")
    dsa.device_status(clear=True)
    got = dsa.dsa_topk(t.cuda(), torch.from_numpy(L).cuda(), k).cpu().numpy()
    exp = oracle_mod.topk(t.float().numpy(), L, k)
    np.testing.assert_array_equal(got, exp)
    assert dsa.device_status() & dsa.STATUS_ERRORS == 0


@pytest.mark.parametrize("seed", range(24))
def test_cluster_random_shapes(oracle_mod, dsa, seed):
    """Seeded random cluster launches: 1-8 rows, strides 200K-700K, lengths
    from 0 to the stride, k from 1 to 2048, fp32 or bf16, and per row one of
    several value patterns (normal, a coarse grid, four levels, mostly -inf,
    sorted either way, a block of large values), so the shared threshold, the
    merge's retry and its tie split meet many combinations."""
    rng = np.random.default_rng(3700 + seed)
    rows = int(rng.integers(1, 9))
    stride = int(rng.integers(200000, 700001))
    k = (2048, 7, 1024, 1, 2048, 512, 2048, 1024)[seed % 8]
    L = rng.integers(0, stride + 1, size=rows).astype(np.int32)
    L[rng.random(rows) < 0.3] = stride
    x = rng.standard_normal((rows, stride)).astype(np.float32)
    for r in range(rows):
        kind = int(rng.integers(0, 7))
        if kind == 1:
            x[r] = np.round(x[r] * 4) / 4
        elif kind == 2:
            x[r] = rng.integers(0, 4, stride).astype(np.float32)
        elif kind == 3:
            keep = rng.random(stride) < 0.001
            x[r] = np.where(keep, x[r], -np.inf)
        elif kind == 4:
            x[r] = np.sort(x[r])
        elif kind == 5:
            x[r] = np.sort(x[r])[::-1]
        elif kind == 6:
            b = int(rng.integers(0, stride - 3000))
            x[r, b:b + 3000] += 40.0
    t = torch.from_numpy(x)
    if seed % 2:
        t = t.to(torch.bfloat16)
    if dsa.plan(rows, stride, k)[0] == 1:
        pytest.skip("this shape takes one CTA per row on this GPU")
    dsa.device_status(clear=True)
    got = dsa.dsa_topk(t.cuda(), torch.from_numpy(L).cuda(), k).cpu().numpy()
    exp = oracle_mod.topk(t.float().numpy(), L, k)
    np.testing.assert_array_equal(got, exp)
    assert dsa.device_status() & dsa.STATUS_ERRORS == 0


@pytest.mark.parametrize("stride_of_run", [1, 2, 3])
@pytest.mark.parametrize("shape", ["rows", "cluster"])
def test_tied_runs_index_cut(oracle_mod, dsa, stride_of_run, shape):
    """A run of one repeated top value: its copies flood the candidate buffer and
    the exact compaction cuts them by index. Dense runs (every position) take the
    dense-range cut (min + need - 1); strided runs take the index select."""
    rng = np.random.default_rng(3100 + stride_of_run)
    if shape == "rows":
        rows, stride, k = 160, 40000, 2048
    else:
        rows, stride, k = 3, 600000, 1024
    x = rng.standard_normal((rows, stride)).astype(np.float32)
    L = np.full(rows, stride, np.int32)
    for r in range(rows):
        a = int(rng.integers(0, stride // 4))
        b = min(stride, a + stride // 2)
        x[r, a:b:stride_of_run] = 7.0 if r % 2 else -np.inf
        if r % 2 == 0:
            x[r, :] = np.where(np.arange(stride) >= a, x[r], -np.inf)  # -inf tail and run, finite head
    L[-1] = stride - 5
    assert (dsa.plan(rows, stride, k)[0] > 1) == (shape == "cluster")
    assert_parity(oracle_mod, dsa, x, L, k)


@pytest.mark.parametrize("k", [1024, 2048])
def test_cluster_rows_mostly_neg_inf(oracle_mod, dsa, k):
    """Cluster ranks with no sampled threshold leave out -inf values; rows with
    fewer than k values above -inf send every rank back over its chunk with no
    threshold. Rows: a few finite values, all -inf, -inf in every other half of
    the chunks, and a normal row with a -inf tail."""
    rng = np.random.default_rng(3300 + k)
    stride = 600000
    L = np.array([stride, stride, stride, stride - 7, 250000], np.int32)
    x = np.full((len(L), stride), -np.inf, np.float32)
    pos = rng.choice(stride, size=500, replace=False)
    x[0, pos] = rng.standard_normal(500).astype(np.float32)
    # row 1: all -inf
    chunk = stride // 16
    for c in range(0, 16, 2):
        x[2, c * chunk:(c + 1) * chunk] = rng.standard_normal(chunk).astype(np.float32)
    x[3, : stride // 2] = rng.standard_normal(stride // 2).astype(np.float32)
    x[4, : 1500] = np.round(rng.standard_normal(1500) * 2).astype(np.float32) / 2
    assert dsa.plan(len(L), stride, k)[0] > 1
    assert_parity(oracle_mod, dsa, x, L, k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_cluster_threshold_shared_by_ranks(oracle_mod, dsa, dtype):
    """Cluster ranks filter with one threshold drawn from every rank's sample.
    Rows where it lies far from a rank's own share: values rising along the
    row (the whole top k in the last chunk), 1000 large values placed between
    two sample runs of one chunk, one chunk of shifted values on a coarse grid
    (ties at the cut), a plain row of another length, a row too short for any
    rank to sample (no threshold: ranks keep every value above -inf) and an
    empty row."""
    import torch
    rng = np.random.default_rng(3500 + (dtype == "bf16"))
    rows, stride, k = 6, 600000, 2048
    L = np.array([stride, stride - 5, stride, 400001, 20000, 0], np.int32)
    x = rng.standard_normal((rows, stride)).astype(np.float32)
    x[0] = np.sort(x[0])
    x[1, 302000:303000] += 50.0  # inside one rank's chunk, clear of its sample runs
    chunk = stride // 16
    x[2, 5 * chunk:6 * chunk] = np.round(rng.standard_normal(chunk) * 4) / 4 + 3.0
    t = torch.from_numpy(x)
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    assert dsa.plan(rows, stride, k)[0] > 1
    dsa.device_status(clear=True)
    got = dsa.dsa_topk(t.cuda(), torch.from_numpy(L).cuda(), k).cpu().numpy()
    exp = oracle_mod.topk(t.float().numpy(), L, k)
    np.testing.assert_array_equal(got, exp)
    assert dsa.device_status() & dsa.STATUS_ERRORS == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("base_offset", [0, 3])
def test_short_rows_kernel(oracle_mod, dsa, dtype, base_offset):
    """Row strides that fit one stage take their own kernel instance, where a
    row with no threshold is copied whole: many rows per CTA (later rows carry
    thresholds), lengths past the 4096-entry handover (a compaction follows
    the copy), ties, special values, an unaligned base."""
    import torch
    rng = np.random.default_rng(3400 + base_offset + (dtype == "bf16"))
    rows, stride, k = 700, 8000, 2048
    L = rng.integers(0, stride + 1, size=rows).astype(np.int32)
    L[:6] = [0, 1, 2048, 4096, 4097, stride]
    x = rng.standard_normal((rows, stride)).astype(np.float32)
    x[1::4] = np.round(x[1::4] * 4) / 4
    x[2, :50] = np.nan
    x[3, 100:200] = np.inf
    t = torch.from_numpy(x)
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    buf = torch.full((base_offset + rows * stride + 8,), float("inf"), dtype=t.dtype)
    buf[base_offset:base_offset + rows * stride] = t.reshape(-1)
    d = buf.cuda()[base_offset:base_offset + rows * stride].view(rows, stride)
    got = dsa.dsa_topk(d, torch.from_numpy(L).cuda(), k).cpu().numpy()
    exp = oracle_mod.topk(t.float().numpy(), L, k)
    np.testing.assert_array_equal(got, exp)
    assert dsa.device_status() & dsa.STATUS_ERRORS == 0


# --------------------------------------------------------- layout and poison
@pytest.mark.parametrize("extra,offset", [(0, 0), (1, 0), (2, 1), (3, 3), (5, 2), (256, 0)])
def test_unaligned_strides_and_bases(oracle_mod, dsa, extra, offset):
    rng = np.random.default_rng(extra * 10 + offset)
    L = np.array([5000, 4096, 17, 9000, 4093, 1, 0, 8195] * 20, np.int32)
    stride = int(L.max()) + extra
    x = rng.standard_normal((len(L), stride)).astype(np.float32)
    assert_parity(oracle_mod, dsa, x, L, 512, base_offset=offset)


@pytest.mark.parametrize("offset", [0, 1, 2, 3])
def test_unaligned_cluster_path(oracle_mod, dsa, offset):
    rng = np.random.default_rng(77 + offset)
    L = np.array([250001, 199999, 250003], np.int32)
    stride = 250003 + offset
    x = rng.standard_normal((3, stride)).astype(np.float32)
    assert_parity(oracle_mod, dsa, x, L, 1024, base_offset=offset)


@pytest.mark.parametrize("poison", [np.inf, np.nan, -np.inf, 3.0e38])
def test_padding_is_never_read(oracle_mod, dsa, poison):
    wl = workloads.make_rows("decode", [0, 1, 2, 3, 4, 5, 6, 7])
    a = np.full_like(wl.logits, poison)
    for i in range(wl.num_rows):
        a[i, :wl.lengths[i]] = wl.logits[i, :wl.lengths[i]]
    base = run_gpu(dsa, wl.logits, wl.lengths, wl.k)
    got = run_gpu(dsa, a, wl.lengths, wl.k)
    np.testing.assert_array_equal(got, base)
    np.testing.assert_array_equal(got, oracle_mod.topk(wl.logits, wl.lengths, wl.k))


def test_stride_invariance_on_gpu(dsa):
    wl = workloads.make_rows("decode", range(16))
    base = run_gpu(dsa, wl.logits, wl.lengths, wl.k)
    Lmax = int(wl.lengths.max())
    for stride in (Lmax, Lmax + 3, 2 * Lmax + 1):
        a = np.ascontiguousarray(wl.logits[:, :Lmax])
        np.testing.assert_array_equal(run_gpu(dsa, a, wl.lengths, wl.k, stride=stride), base)


def test_lengths_are_clamped(oracle_mod, dsa):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 3000)).astype(np.float32)
    L = np.array([-5, 0, 3000, 3001, 2 ** 31 - 1, 1500], np.int32)
    assert_parity(oracle_mod, dsa, x, L, 256)


# ------------------------------------------------------------ value patterns
def _special_rows(rng, rows, width):
    pool = np.array([np.nan, np.inf, -np.inf, 0.0, -0.0, 1.0, -1.0, 2.5], np.float32)
    x = rng.standard_normal((rows, width)).astype(np.float32)
    mask = rng.random((rows, width)) < 0.05
    x[mask] = pool[rng.integers(0, len(pool), mask.sum())]
    return x


def test_special_values(oracle_mod, dsa):
    rng = np.random.default_rng(8)
    x = _special_rows(rng, 200, 9000)
    x[3, :] = np.nan
    x[4, :] = -np.inf
    x[5, :] = -0.0
    x[6, ::2] = 0.0
    x[7, :] = np.inf
    L = rng.integers(0, 9001, 200).astype(np.int32)
    L[3:8] = 9000
    assert_parity(oracle_mod, dsa, x, L, 2048)


def test_special_values_cluster(oracle_mod, dsa):
    rng = np.random.default_rng(9)
    x = _special_rows(rng, 3, 200000)
    x[1, 150000:] = np.nan
    x[2, :] = -0.0
    x[2, 199990] = 0.0
    L = np.array([200000, 200000, 200000], np.int32)
    assert_parity(oracle_mod, dsa, x, L, 1024)


@pytest.mark.parametrize("pattern", ["increasing", "decreasing", "all_equal", "two_levels", "sawtooth"])
@pytest.mark.parametrize("rows", [160, 3])
def test_adversarial_orders(oracle_mod, dsa, pattern, rows):
    width = 150000 if rows == 3 else 40000
    j = np.arange(width, dtype=np.float64)
    if pattern == "increasing":
        row = j
    elif pattern == "decreasing":
        row = -j
    elif pattern == "all_equal":
        row = np.zeros(width)
    elif pattern == "two_levels":
        row = (j % 7 == 0).astype(np.float64)
    else:
        row = j % 5000
    x = np.tile(row.astype(np.float32), (rows, 1))
    L = np.full(rows, width, np.int32)
    L[::2] = width - 7
    assert_parity(oracle_mod, dsa, x, L, 2048)


@pytest.mark.parametrize("k", [2048, 512])
def test_fp8_grid_many_rows(oracle_mod, dsa, k):
    """Many rows of values on the fp8 e4m3 grid (heavy ties at every level):
    the many-row path with its estimates carried between rows, and the
    finisher's sorted fallback for buckets full of equal keys."""
    rng = np.random.default_rng(77 + k)
    rows, width = 296, 65536
    x = workloads.round_to_e4m3(rng.standard_normal((rows, width))).astype(np.float32)
    L = rng.integers(30000, width, size=rows, endpoint=True).astype(np.int32)
    assert_parity(oracle_mod, dsa, x, L, k)


def test_few_levels_many_rows(oracle_mod, dsa):
    """Three distinct values over many rows: every bucket of the finisher's
    first pass is one level, so the sorted fallback orders them by index."""
    rng = np.random.default_rng(31)
    x = (rng.integers(0, 3, (160, 50000)) * 1.0).astype(np.float32)
    L = np.full(160, 50000, np.int32)
    L[1::3] = 33333
    assert_parity(oracle_mod, dsa, x, L, 2048)
    assert_parity(oracle_mod, dsa, x, L, 100)


SAMPLE_RUNS = 32    # a row's first threshold is sampled from 32 runs of 128 values,
FEW_ROWS_SAMPLE_RUNS = 16  # or 16 when every CTA has at most two rows
CLUSTER_SAMPLE_RUNS = 8  # a cluster rank's from 8 (one per filter warp)
CHUNK_ALIGN = 8     # a cluster rank's chunk is rounded up to a multiple of 8 elements


def _sample_runs(span, runs):
    """Start offsets of the evenly spaced 128-value runs a first threshold is
    sampled from (16-byte aligned rows and chunks)."""
    return [((span - 128) * r // (runs - 1)) & ~3 for r in range(runs)]


def test_sampled_threshold_fallback_many_rows(oracle_mod, dsa):
    """Large values exactly where a row's first threshold is sampled, small
    values elsewhere: the sampled threshold lets far fewer than k values
    through, so the row must be re-read with no threshold, and the result must
    still be exact."""
    rng = np.random.default_rng(5)
    rows, L, stride = 148, 120000, 131072  # one row per CTA: every row is a first row
    x = (rng.standard_normal((rows, stride)) * 0.01).astype(np.float32)
    for b in sorted(set(_sample_runs(L, SAMPLE_RUNS)) | set(_sample_runs(L, FEW_ROWS_SAMPLE_RUNS))):
        x[:, b:b + 128] = 100.0 + rng.random((rows, 128), dtype=np.float32)
    Ls = np.full(rows, L, np.int32)
    dsa.device_status(clear=True)
    assert_parity(oracle_mod, dsa, x, Ls, 2048)
    st = dsa.device_status()
    assert st & dsa.STATUS_ERRORS == 0 and st & dsa.STATUS_REREAD, st


def test_carried_estimate_overshoot_many_rows(oracle_mod, dsa):
    """Four or more rows per CTA whose values drop by 3 from one of a CTA's
    rows to its next, with lengths within 1/8 of each other: the threshold
    carried from a CTA's earlier rows (the finisher's estimate two rows back,
    or the filter's own bound one row back) lets almost nothing through, so
    every row after a CTA's first is re-read from global memory. Every row is
    compared; a third of the rows sit on a coarse grid so the re-read also
    resolves ties."""
    k, stride = 2048, 52224
    grid = dsa.plan(148 * 5, stride, k)[1]
    rows = 5 * grid  # rows r, r+grid, ... go to the same CTA, in order
    rng = np.random.default_rng(404)
    L = rng.integers(50000, 52000, size=rows, endpoint=True).astype(np.int32)
    x = rng.standard_normal((rows, stride)).astype(np.float32)
    x[2::3] = np.round(x[2::3] * 4) / 4
    h = (np.arange(rows) // grid).astype(np.float32)  # the row's position in its CTA's sequence
    x -= 3.0 * h[:, None]
    assert dsa.plan(rows, stride, k) == (1, grid)
    dsa.device_status(clear=True)
    assert_parity(oracle_mod, dsa, x, L, k)
    st = dsa.device_status()
    assert st & dsa.STATUS_ERRORS == 0 and st & dsa.STATUS_REREAD, st


def test_sampled_threshold_fallback_cluster(oracle_mod, dsa):
    """The same trap for the cluster path: every rank's sample lands on large
    values, so every rank must re-read its chunk."""
    rng = np.random.default_rng(6)
    rows, L, stride, ranks = 4, 900000, 900096, 16
    if dsa.plan(rows, stride, 1024)[0] != ranks:
        pytest.skip("this GPU does not run 16-CTA clusters")
    chunk = (-(-L // ranks) + CHUNK_ALIGN - 1) // CHUNK_ALIGN * CHUNK_ALIGN
    x = (rng.standard_normal((rows, stride)) * 0.01).astype(np.float32)
    for r in range(ranks):
        c0, c1 = min(L, r * chunk), min(L, r * chunk + chunk)
        for b in _sample_runs(c1 - c0, CLUSTER_SAMPLE_RUNS):
            x[:, c0 + b:c0 + b + 128] = 100.0 + rng.random((rows, 128), dtype=np.float32)
    Ls = np.full(rows, L, np.int32)
    dsa.device_status(clear=True)
    assert_parity(oracle_mod, dsa, x, Ls, 1024)
    st = dsa.device_status()
    assert st & dsa.STATUS_ERRORS == 0 and st & dsa.STATUS_REREAD, st


def test_heavy_ties_cluster_exact_path(oracle_mod, dsa):
    """Few levels across a cluster-split row: the merge must split the tied
    threshold level across ranks in index order."""
    rng = np.random.default_rng(12)
    x = (rng.integers(0, 3, (4, 400000)) * 1.0).astype(np.float32)
    L = np.array([400000, 399999, 262145, 400000], np.int32)
    assert_parity(oracle_mod, dsa, x, L, 2048)
    assert_parity(oracle_mod, dsa, x, L, 7)


# ------------------------------------------------------------ execution model
def test_repeat_calls_are_deterministic(dsa):
    wl = workloads.make("decode")
    a = run_gpu(dsa, wl.logits, wl.lengths, wl.k)
    for _ in range(3):
        np.testing.assert_array_equal(run_gpu(dsa, wl.logits, wl.lengths, wl.k), a)


def test_cuda_graph_replay(oracle_mod, dsa):
    wl = workloads.make("decode")
    logits = torch.from_numpy(wl.logits).cuda()
    lengths = torch.from_numpy(wl.lengths).cuda()
    out = torch.empty((wl.num_rows, wl.k), dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dsa.dsa_topk(logits, lengths, wl.k, out=out)  # uncaptured first call (attributes)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(3):
            dsa.dsa_topk(logits, lengths, wl.k, out=out)
    exp = oracle_mod.topk(wl.logits, wl.lengths, wl.k)
    for _ in range(5):
        out.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out.cpu().numpy(), exp)
    del g


def test_torch_binding_uses_stride0(oracle_mod, dsa):
    """A sliced (non-contiguous) view is read at its row stride."""
    wl = workloads.make_rows("tiny", range(4))
    full = torch.from_numpy(wl.logits).cuda()          # [4, 4096]
    view = full[:, :4000]                               # stride(0) = 4096, size(1) = 4000
    assert view.stride(0) == 4096 and not view.is_contiguous()
    out = dsa.dsa_topk(view, torch.from_numpy(wl.lengths).cuda(), wl.k)
    np.testing.assert_array_equal(out.cpu().numpy(), oracle_mod.topk(wl.logits, wl.lengths, wl.k))


def test_host_buffer_entry_point(oracle_mod, dsa):
    wl = workloads.make("tiny")
    h_logits = torch.from_numpy(wl.logits).pin_memory()
    h_len = torch.from_numpy(wl.lengths).pin_memory()
    h_out = torch.empty((wl.num_rows, wl.k), dtype=torch.int32).pin_memory()
    d_logits = torch.empty(wl.logits.size, dtype=torch.float32, device="cuda")
    d_len = torch.empty(wl.num_rows, dtype=torch.int32, device="cuda")
    d_out = torch.empty(wl.num_rows * wl.k, dtype=torch.int32, device="cuda")
    dsa.dsa_topk_host(h_logits, h_len, wl.k, h_out, d_logits, d_len, d_out)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(h_out.numpy(), oracle_mod.topk(wl.logits, wl.lengths, wl.k))


def test_mixed_paths_in_one_graph(oracle_mod, dsa):
    """Back-to-back dependent launches of both kernels in one CUDA graph
    (programmatic dependent launch between them): every output is exact after
    every replay."""
    a = workloads.make_rows("tiny", range(4))
    b = workloads.make_rows("decode", range(16))
    ta, la = torch.from_numpy(a.logits).cuda(), torch.from_numpy(a.lengths).cuda()
    tb, lb = torch.from_numpy(b.logits).cuda(), torch.from_numpy(b.lengths).cuda()
    oa = torch.empty((4, a.k), dtype=torch.int32, device="cuda")
    ob = torch.empty((16, b.k), dtype=torch.int32, device="cuda")
    assert dsa.plan(16, b.row_stride, b.k)[0] > 1 and dsa.plan(4, a.row_stride, a.k)[0] == 1
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dsa.dsa_topk(ta, la, a.k, out=oa)
        dsa.dsa_topk(tb, lb, b.k, out=ob)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(4):
            dsa.dsa_topk(ta, la, a.k, out=oa)
            dsa.dsa_topk(tb, lb, b.k, out=ob)
    ea, eb = oracle_mod.topk(a.logits, a.lengths, a.k), oracle_mod.topk(b.logits, b.lengths, b.k)
    for _ in range(3):
        oa.fill_(-7)
        ob.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(oa.cpu().numpy(), ea)
        np.testing.assert_array_equal(ob.cpu().numpy(), eb)
    del g


def _timed_call(dsa, logits, lengths, k):
    import time
    out = torch.empty((logits.shape[0], k), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    dsa.dsa_topk(logits, lengths, k, out=out)
    torch.cuda.synchronize()
    return out, time.perf_counter() - t0


@pytest.mark.parametrize("path", ["rows", "cluster"])
def test_wait_timeout_ends_the_call(oracle_mod, dsa, path):
    """A test hook makes every CTA's producer leave one stage unissued, so the
    consumers' wait for it runs out (limit 50 ms). The call must return within
    a few limits with the timeout bit set, and the next call, hooks reset,
    must be exact. Nothing faults: the skipped stage has no copy in flight."""
    rng = np.random.default_rng(61)
    if path == "rows":
        rows, width = 296, 60000     # 8 stages per row: stage 2 is inside each CTA's first row
    else:
        rows, width = 3, 200000      # a cluster per row, several stages per rank
    x = torch.from_numpy(rng.standard_normal((rows, width)).astype(np.float32)).cuda()
    L = torch.full((rows,), width, dtype=torch.int32, device="cuda")
    assert (dsa.plan(rows, width, 1024)[0] > 1) == (path == "cluster")
    dsa.device_status(clear=True)
    try:
        dsa.set_test_hooks(wait_limit_ns=50_000_000, skip_stage=2)
        out, dt = _timed_call(dsa, x, L, 1024)
        st = dsa.device_status(clear=True)
    finally:
        dsa.set_test_hooks()  # defaults
    assert st & dsa.STATUS_WAIT_TIMEOUT, st
    assert dt < 2.0, "the aborted call took %.3f s" % dt
    if path == "cluster":
        assert bool((out == -1).all()), "rows of a cluster that gave up are written as -1"
    out, dt = _timed_call(dsa, x, L, 1024)
    np.testing.assert_array_equal(out.cpu().numpy(), oracle_mod.topk(x.cpu().numpy(), L.cpu().numpy(), 1024))
    assert dsa.device_status(clear=True) & dsa.STATUS_ERRORS == 0


def test_no_device_side_errors(dsa):
    assert dsa.device_status() & dsa.STATUS_ERRORS == 0
