"""Multi-rank runs of the multi-GPU host logic over gloo on the CPU.

Rows are independent. Two modes exist: replicas (each rank its own batch)
and row shards (one batch split into contiguous row blocks, one per rank,
``sparse_attention_indexer_strided_b200.shard``). Neither has a data-path
collective; the exchanges are the max over ranks of the timed duration and
an optional all-gather of the results. These tests run them with real
process-group ranks (no GPU needed); the oracle stands in for each rank's
top-k call, since what is checked here is the partition and the gather.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, queue):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        dist.barrier()
        ms_max = bench.max_over_ranks(local_ms[rank], dist, "cpu")
        value = bench.job_rows_per_s(world, 4096, 10, ms_max)
        queue.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


def _shard_main(rank, world, port, config, queue):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import numpy as np
    import oracle
    import workloads
    from sparse_attention_indexer_strided_b200 import shard
    try:
        n = workloads.spec(config).num_rows
        r0, r1 = shard.row_block(n, world, rank)
        wl = workloads.make_rows(config, range(r0, r1))  # this rank holds its own rows only
        block = torch.from_numpy(oracle.topk(wl.logits, wl.lengths, wl.k, threads=1))
        full = shard.gather_rows(block, n, world, rank)
        queue.put((rank, r0, r1, full.numpy()))
    finally:
        dist.destroy_process_group()


def _run(world, local_ms, target=None, args=None):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    target = target or _rank_main
    procs = [ctx.Process(target=target, args=(r, world, port) + tuple(args if args is not None else (local_ms,))
                         + (queue,)) for r in range(world)]
    for p in procs:
        p.start()
    results = [queue.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(results)


def test_two_ranks_take_the_slowest_duration():
    res = _run(2, [6.0, 7.5])
    assert [r for r, _, _ in res] == [0, 1]
    for _, ms_max, value in res:
        assert ms_max == pytest.approx(7.5)
        # 2 ranks x 4096 rows x 10 steps over the slowest rank's 7.5 ms
        assert value == pytest.approx(2 * 4096 * 10 / 7.5e-3)


def test_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, None) == 3.25
    assert bench.job_rows_per_s(1, 4096, 200, 124.0) == pytest.approx(4096 * 200 / 0.124)


def test_row_blocks_partition_the_batch():
    sys.path.insert(0, ROOT)
    from sparse_attention_indexer_strided_b200 import shard
    for n in (0, 1, 4, 64, 255, 4096):
        for world in (1, 2, 3, 8):
            blocks = [shard.row_block(n, world, r) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == n
            assert all(blocks[i][1] == blocks[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1 and max(sizes) == shard.max_block(n, world)
    with pytest.raises(ValueError):
        shard.row_block(4, 2, 2)


@pytest.mark.parametrize("world", [2, 3])
def test_row_shards_gathered_equal_the_whole_batch(oracle_mod, world):
    """Each rank takes its row block of the decode batch (64 rows; uneven
    blocks for 3 ranks), computes it, and the all-gather reassembles exactly
    the whole batch's result on every rank."""
    import workloads
    res = _run(world, None, target=_shard_main, args=("decode",))
    wl = workloads.make("decode")
    exp = oracle_mod.topk(wl.logits, wl.lengths, wl.k)
    covered = np.zeros(wl.num_rows, np.int32)
    for rank, r0, r1, full in res:
        covered[r0:r1] += 1
        np.testing.assert_array_equal(full, exp)
    assert np.all(covered == 1)
