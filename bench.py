#!/usr/bin/env python
"""Benchmark of the strided indexer top-k on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config prefill|ties|decode|cluster|tiny] [--no-per-config]

One step = one ``dsa_topk`` call over the whole batch of the chosen workload
(default: prefill, 4096 rows of a 131072-token causal context, k=2048), with
the inputs already resident in HBM. The prefill input (2.15 GB) is larger than
the 126 MB L2, so consecutive steps read HBM; no flush is needed.

Prints one JSON line (rank 0). ``value`` is rows/s over all ranks. By default
every rank processes its own copy of the batch (weak scaling). With
``--shard rows`` one batch is split into contiguous row blocks, one per rank,
each rank holding only its own rows (strong scaling). Neither mode has a
collective on the data path, only the max-over-ranks reduction of the timings. The line also carries
the HBM roofline of the kernel, the oracle's CPU throughput on a bounded sample
(N=1), the host-buffer end-to-end throughput, SM clocks sampled during the
timed region, and per-workload timings of all five workloads (N=1).

``--impl reference`` times the CPU oracle instead (rank 0 only), each step a
bounded sample of rows of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "top-k rows/s and achieved HBM GB/s (fraction of B200 peak) per config"
L2_BYTES = 126 * 1024 * 1024
DESCRIPTIONS = {
    "tiny": "tiny: 4 rows x L=4000 (row stride 4096), k=512, fp32 N(0,1)",
    "decode": "decode: 64 rows, L_i ~ U[1,65536] (row stride 65536), k=2048, N(0,1) on the fp8-e4m3 grid",
    "cluster": "cluster: 4 rows x L=900000 (row stride 900096), k=1024, N(0,1) with -inf last 10%",
    "prefill": "prefill: 4096 rows, L_i=126977+i (row stride 131072), k=2048, N(0,1)+0.5*log1p(distance)",
    "ties": "ties: 256 rows x L=131072 (row stride 131328), k=2048, 16 fp32 levels",
}


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", choices=list(workloads.CONFIG_NAMES), default="prefill")
    p.add_argument("--no-per-config", action="store_true", help="skip the five-workload table")
    p.add_argument("--e2e-steps", type=int, default=5, help="0 skips the host-buffer run")
    p.add_argument("--rows", type=int, default=0, help="use only the first N rows (profiling runs)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--shard", choices=["none", "rows"], default="none",
                   help="rows: split one batch into contiguous row blocks across ranks (strong scaling)")
    return p.parse_args()


def load_workload(config, rows=0):
    if rows and rows < workloads.spec(config).num_rows:
        return workloads.make_rows(config, range(rows))
    return workloads.make(config)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    return 6650.0, "fallback (6.65 TB/s, earlier measurement on this pool)"


def _code_only(text):
    """Source text without comments and blank lines (the digest follows code)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = []
    for line in text.splitlines():
        line = re.sub(r"//.*$", "", line).rstrip()
        if line.strip():
            lines.append(line)
    return "\n".join(lines)


def source_sha():
    """Digest of the code of every kernel source file (a traffic figure is only
    valid for it); comment-only edits keep it."""
    csrc = os.path.join(ROOT, "sparse_attention_indexer_strided_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            h.update(name.encode())
            h.update(_code_only(open(os.path.join(csrc, name), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(config):
    """DRAM bytes per launch from the committed ncu summary of this workload,
    or None when it is missing or was taken on another kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic_%s.txt" % config)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_sha = re.search(r"^source_sha256_16:\s*(\w+)", text, re.M)
    m_b = re.search(r"^dram_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    if not (m_sha and m_b) or m_sha.group(1) != source_sha():
        return None
    return float(m_b.group(1))


# ------------------------------------------------------------ rank logic
def max_over_ranks(ms, dist=None, device="cpu"):
    """The slowest rank's duration: every rank's timed region ends when all
    have finished, so whole-job throughput divides by this."""
    if dist is None:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rows_per_s(world, rows_per_rank, steps, ms_max):
    """Rows of all ranks per second (weak scaling: each rank its own batch)."""
    return world * rows_per_rank * steps / (ms_max / 1e3)


def sharded_rows_per_s(batch_rows, steps, ms_max):
    """Rows of one batch split across ranks, per second of the slowest rank."""
    return batch_rows * steps / (ms_max / 1e3)


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons via NVML (read-only) on a
    background thread while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, local_index):
        self.samples, self.reasons, self.max_mhz, self.ok = [], 0, None, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [t for t in vis.split(",") if t.strip()]
            idx = int(ids[local_index]) if ids and ids[local_index].strip().isdigit() else local_index
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _reasons(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(f(self.h))

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self._reasons()
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": sorted(names),
                "samples": len(self.samples)}


# --------------------------------------------------------------- GPU timing
def time_graph(dsa, torch, calls, reps=5):
    """Capture `calls` (list of zero-arg launches) in one CUDA graph, replay
    `reps` times; returns the median microseconds per call."""
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for c in calls[:2]:
            c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for c in calls:
            c()
    with torch.cuda.stream(s):
        g.replay()
    torch.cuda.synchronize()
    out = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):  # replay() launches on the current stream
            e0.record(s)
            g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1) * 1e3 / len(calls))
    del g
    return statistics.median(out)


def _time_workload(dsa, torch, peak, wl, dtype=None, unsorted=False, table=False):
    """CUDA-graph timing of one workload (rotating input copies whose total
    exceeds 4x L2, so each call reads HBM), plus an L2-warm number."""
    elem = 4 if dtype is None else 2
    vb = workloads.valid_bytes(wl.lengths) * elem // 4
    base = torch.from_numpy(wl.logits).cuda()
    if dtype is not None:
        base = base.to(dtype)
    tensor_bytes = base.numel() * base.element_size()
    R = max(1, min(64, -(-4 * L2_BYTES // tensor_bytes)))
    copies = [base] + [base.clone() for _ in range(R - 1)]
    lengths = torch.from_numpy(wl.lengths).cuda()
    out = torch.empty((wl.num_rows, wl.k), dtype=torch.int32, device="cuda")
    tab = None
    if table:  # a per-row lookup table (row-local index -> int32 value), made on the device
        tab = torch.randint(0, 1 << 30, (wl.num_rows, wl.row_stride), dtype=torch.int32, device="cuda")
    kw = {"unsorted": unsorted, "index_table": tab}
    n_calls = max(R, min(256, max(8, int(2e9 // max(vb, 1)))))
    cold = [(lambda c=copies[i % R]: dsa.dsa_topk(c, lengths, wl.k, out=out, **kw)) for i in range(n_calls)]
    dsa.device_status(clear=True)
    us_cold = time_graph(dsa, torch, cold)
    warm = [(lambda: dsa.dsa_topk(base, lengths, wl.k, out=out, **kw)) for _ in range(min(n_calls, 64))]
    us_warm = time_graph(dsa, torch, warm)
    status = dsa.device_status(clear=True)
    cs, grid = dsa.plan(wl.num_rows, wl.row_stride, wl.k)
    gbs = vb / us_cold / 1e3
    res = {
        "us_per_call": round(us_cold, 3), "rows_per_s": round(wl.num_rows / us_cold * 1e6, 1),
        "valid_gbs": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4),
        "us_per_call_warm_l2": round(us_warm, 3), "valid_bytes": vb,
        "rotating_copies": R, "cluster_size": cs, "grid": grid,
        "device_status": status,  # bit 2: some row was re-read after a speculative threshold (info)
    }
    del copies, base, out, tab
    torch.cuda.empty_cache()
    return res


def per_config_table(dsa, torch, peak):
    """All five workloads, then the prefill workload with each call option:
    bf16 logits (2 bytes per valid logit), the unsorted (set) output, and an
    index table applied to every output."""
    rows = {}
    for name in workloads.CONFIG_NAMES:
        rows[name] = _time_workload(dsa, torch, peak, workloads.make(name))
    wl = workloads.make("prefill")
    rows["prefill_bf16"] = _time_workload(dsa, torch, peak, wl, dtype=torch.bfloat16)
    rows["prefill_unsorted"] = _time_workload(dsa, torch, peak, wl, unsorted=True)
    rows["prefill_index_table"] = _time_workload(dsa, torch, peak, wl, table=True)
    return rows


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        print("warning: --gpus %d but WORLD_SIZE=%d" % (args.gpus, world), file=sys.stderr)
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    import sparse_attention_indexer_strided_b200 as dsa

    peak, peak_src = load_peaks()
    if args.shard == "rows":
        from sparse_attention_indexer_strided_b200 import shard
        batch_rows = args.rows or workloads.spec(args.config).num_rows
        r0, r1 = shard.row_block(batch_rows, world, rank)
        wl = workloads.make_rows(args.config, range(r0, r1))  # this rank's rows only
    else:
        wl = load_workload(args.config, args.rows)
    vb = workloads.valid_bytes(wl.lengths)
    logits = torch.from_numpy(wl.logits).cuda()
    lengths = torch.from_numpy(wl.lengths).cuda()
    out = torch.empty((wl.num_rows, wl.k), dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()
    cs, grid = dsa.plan(wl.num_rows, wl.row_stride, wl.k)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            dsa.dsa_topk(logits, lengths, wl.k, out=out, stream=stream)
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps, one kernel launch each. The K calls
    # go to the GPU as one CUDA graph captured beforehand, as a serving loop
    # replays a fixed step; the replay is the only thing timed.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(args.steps):
            dsa.dsa_topk(logits, lengths, wl.k, out=out, stream=stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        with torch.cuda.stream(stream):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    del graph
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, dist if world > 1 else None, "cuda")
    status = dsa.device_status()

    # ---- end to end through the host-buffer C-ABI entry point
    e2e = None
    if args.e2e_steps > 0:
        e2e = run_e2e(args, dsa, torch, dist, wl, logits, lengths, out, stream, world,
                      batch_rows if args.shard == "rows" else None)

    per_launch_us = ms / args.steps * 1e3
    achieved = vb / per_launch_us / 1e3  # GB/s of valid logits
    if args.shard == "rows":
        value = sharded_rows_per_s(batch_rows, args.steps, ms_max)
        parallelism = "rows%d (one batch in contiguous row blocks, no data-path collective)" % world
    else:
        value = job_rows_per_s(world, wl.num_rows, args.steps, ms_max)
        parallelism = "dp%d (each GPU its own batch, no data-path collective)" % world
    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "rows/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True,
        "scaling": "strong" if args.shard == "rows" else "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": DESCRIPTIONS[args.config],
            "num_rows": wl.num_rows, "row_stride": wl.row_stride, "k": wl.k,
            "valid_bytes_per_step": vb,
            "l2": ("inputs %.2f GB > 126 MB L2, no flush needed" % (wl.logits.nbytes / 1e9)
                   if wl.logits.nbytes > 4 * L2_BYTES else "inputs smaller than L2: numbers are L2-warm"),
            "parallelism": parallelism,
            "launch": {"cluster_size": cs, "grid": grid, "timed_as": "one CUDA graph of the K calls, replayed once"},
            "input_sha256_16": workloads.sha256(wl.logits)[:16],
        },
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": profiled_traffic(args.config),
            "peak_source": peak_src, "kernel": "topk_rows_kernel" if cs == 1 else "topk_cluster_kernel",
            "algorithmic_bytes_per_launch": vb,
        },
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "device_status": status,
    }
    if world == 1 and rank == 0:
        if not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(args.config)
        if not args.no_per_config:
            del logits, out
            torch.cuda.empty_cache()
            result["per_config"] = per_config_table(dsa, torch, peak)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_e2e(args, dsa, torch, dist, wl, logits, lengths, out, stream, world, batch_rows=None):
    """Same metric through dsa_topk_host: pinned host inputs copied in and the
    result copied out inside the timed region, every step. ``batch_rows``: row
    shards of one batch (rows/s of that batch); None: one batch per rank.
    Bytes per step are whole-job figures (all ranks)."""
    h_logits = torch.from_numpy(wl.logits).pin_memory()
    h_len = torch.from_numpy(wl.lengths).pin_memory()
    h_out = torch.empty((wl.num_rows, wl.k), dtype=torch.int32).pin_memory()
    d_out_flat = out.view(-1)
    for _ in range(2):
        dsa.dsa_topk_host(h_logits, h_len, wl.k, h_out, logits.view(-1), lengths, d_out_flat, stream=stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.e2e_steps):
        dsa.dsa_topk_host(h_logits, h_len, wl.k, h_out, logits.view(-1), lengths, d_out_flat, stream=stream)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = torch.tensor([f0.elapsed_time(f1)], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
    sec = float(e2e_ms.item()) / 1e3
    io = torch.tensor([float(wl.logits.nbytes + wl.lengths.nbytes), float(wl.num_rows * wl.k * 4)],
                      dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(io, op=dist.ReduceOp.SUM)
    rows = batch_rows if batch_rows is not None else world * wl.num_rows
    return {"value": round(rows * args.e2e_steps / sec, 1), "unit": "rows/s",
            "h2d_bytes_per_step": int(io[0].item()), "d2h_bytes_per_step": int(io[1].item()),
            "steps": args.e2e_steps, "api": "dsa_topk_host (C ABI, pinned host buffers)"}


def oracle_sample_rows(config, n_rows, offset=0):
    s = workloads.spec(config)
    stride = max(1, s.num_rows // n_rows)
    return [(offset + i * stride) % s.num_rows for i in range(min(n_rows, s.num_rows))]


def cpu_baseline(config):
    import oracle

    oracle.build()
    rows = oracle_sample_rows(config, 1024)
    wl = workloads.make_rows(config, rows)
    t0 = time.perf_counter()
    oracle.topk(wl.logits, wl.lengths, wl.k, threads=0)
    dt = time.perf_counter() - t0
    return {"value": round(len(rows) / dt, 1), "unit": "rows/s", "cores": oracle.hardware_threads(),
            "kind": "oracle",
            "sample": "%d of %d %s rows (evenly spaced), std::stable_sort per row on all host threads, %.2f s wall"
                      % (len(rows), workloads.spec(config).num_rows, config, dt)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    oracle.build()
    s = workloads.spec(args.config)
    per_step = min(s.num_rows, 64)
    times = []
    for step in range(args.warmup + args.steps):
        rows = oracle_sample_rows(args.config, per_step, offset=step)
        wl = workloads.make_rows(args.config, rows)
        t0 = time.perf_counter()
        oracle.topk(wl.logits, wl.lengths, wl.k, threads=0)
        if step >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = per_step * len(times) / total
    print(json.dumps({
        "impl": "reference",
        "metric": METRIC, "value": round(value, 1), "unit": "rows/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / len(times) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": DESCRIPTIONS[args.config], "num_rows": s.num_rows, "row_stride": s.row_stride,
                   "k": s.k, "sample_rows_per_step": per_step},
        "cpu_baseline": {"value": round(value, 1), "unit": "rows/s", "cores": oracle.hardware_threads(),
                         "kind": "oracle",
                         "sample": "%d evenly spaced %s rows per step (full rows), all host threads"
                                   % (per_step, args.config)},
        "e2e": {"value": round(value, 1), "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
