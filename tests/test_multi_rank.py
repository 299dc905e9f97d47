"""World-size-2 runs of the multi-GPU bookkeeping over gloo on the CPU.

Rows are independent, so each rank runs its own batch with no data-path
collective; the only exchange is the max over ranks of the timed duration.
These tests check that exchange and the whole-job aggregate with two real
process-group ranks (no GPU needed).
"""
import os
import socket
import sys

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


def _run(world, local_ms):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, queue)) for r in range(world)]
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
