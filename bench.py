#!/usr/bin/env python
"""Throughput of one CSA2 decode group step over an FP4 main KV on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 2]

A step is one pass of the whole hot path over one batch: quantise the
step's new main-KV entries into the FP4 cache, then every layer of the
group in order (index scan + top-K for Full / Reindex / pool-Reindex
layers, sparse MQA attention for every layer), through one
csa2_group_decode call.  Default workload: the decoder group Full,
Reindex, Reindex, Reuse at 131,072 entries (128K tokens, r=1), batch 4.

Prints one JSON line (rank 0).  value = queries/s over all ranks (a query
is one (row, position) carried through every layer), measured with CUDA
events on the launching stream, max over ranks, caches resident in HBM,
L2 flushed (256 MB memset) between steps outside the timed events.
Under torchrun each rank runs its own copy of the workload (batch rows
are independent sequences: no collective on the data path).
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp4_kv_cache_mxfp4_b200 import build as _build  # noqa: E402
from fp4_kv_cache_mxfp4_b200 import workloads  # noqa: E402
from fp4_kv_cache_mxfp4_b200.device_workload import make_device_workload  # noqa: E402

METRIC = "CSA2 decode queries/s and HBM GB/s vs peak at 128K ctx, FP4 main KV"
UNIT = "queries/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0

# DRAM traffic (read + write) of one index_scan_kernel launch of the
# default workload, from an ncu capture of that kernel (profiles/), valid
# only while the scan's sources hash to the recorded value.
SCAN_TRAFFIC = {"sha": "cf0057f69f76fa80", "bytes_per_launch": 138266880}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=2)
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (barrier and max-reduction only)
# ---------------------------------------------------------------------------

def dist_setup(backend="nccl"):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE).
    Ranks are replicas: each runs its own batch rows, and the only traffic
    between them is the barrier and the max-reduction of timings."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if backend == "nccl":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                                 device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """The slowest rank's figure (every rank gets it)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_queries_per_s(queries_per_rank, world, max_ms_per_step):
    """Whole-job throughput: every rank's queries over the slowest rank's
    step time (weak scaling: the work per rank is fixed)."""
    return queries_per_rank * world / (max_ms_per_step * 1e-3)


# ---------------------------------------------------------------------------
# clocks during the run
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, line in self.lines:
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1])); smax.append(float(p[2])); power.append(float(p[3]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------------
# algorithmic bytes
# ---------------------------------------------------------------------------

def scan_algorithmic_bytes(wl):
    """Bytes one index_scan_kernel launch must move (Full / Reindex scan):
    index-K rows once, one fp32 score per (query, entry), index-Q and w."""
    per_row = wl.N * 128 * 2 + wl.Q * wl.N * 4 + wl.Q * (32 * 128 * 2 + 32 * 4)
    return wl.B * per_row


def step_algorithmic_bytes(wl):
    """Algorithmic HBM bytes of one whole step (same accounting as the
    per-kernel figures): the scans, the new entries (read bf16, write FP4),
    and per layer the gathered FP4 entries, the window, q and the output."""
    n_index = sum(1 for m in wl.modes if m in (workloads.FULL, workloads.REINDEX))
    total = n_index * scan_algorithmic_bytes(wl)
    total += wl.B * wl.n_new * (1024 + 288)
    per_query_attn = wl.K * 288 + wl.W * 1024 + 64 * 512 * 2 * 2
    total += len(wl.modes) * wl.B * wl.Q * per_query_attn
    return total


def kernel_source_sha():
    h = hashlib.sha256()
    for f in ("common.cuh", "index_scan.cuh"):
        h.update(open(os.path.join(ROOT, "fp4_kv_cache_mxfp4_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Sustained bf16 TFLOP/s: the prefill scan runs inside a long step."""
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def scan_algorithmic_flops(wl):
    """Flops of one index_scan_kernel launch: 32 heads x 128 dims x 2 per
    (query, visible entry)."""
    return wl.B * sum(wl.n_vis) * 32 * 128 * 2


# ---------------------------------------------------------------------------
# the oracle as CPU baseline / reference arm
# ---------------------------------------------------------------------------

ORACLE_MAX_QUERIES = 8


def oracle_query_sample(wl):
    """Queries of a batch row the oracle runs per step: all of them up to
    ORACLE_MAX_QUERIES, else the last ORACLE_MAX_QUERIES of the chunk (the
    longest visible prefixes, so the sample is the costliest slice)."""
    if wl.Q <= ORACLE_MAX_QUERIES:
        return 0, wl.Q
    return wl.Q - ORACLE_MAX_QUERIES, ORACLE_MAX_QUERIES


def oracle_row_setup(wl, b):
    """Host inputs of batch row b for the oracle, restricted to the sampled
    queries: its FP4 cache built by the oracle's own quantiser (only the rows
    the oracle's layers will read are filled: attention reads nothing else),
    index-K and the sampled queries' layer inputs and windows."""
    from oracle import fp4, group, indexer
    q0, qn = oracle_query_sample(wl)
    x = workloads.main_kv_rows(wl, b, 0, wl.N).float().numpy()
    kI = workloads.index_k(wl, b).float().numpy()
    n_vis = np.array(wl.n_vis[q0:q0 + qn])
    w0, w1 = q0 * wl.swa_step, (q0 + qn - 1) * wl.swa_step + wl.W
    layers = []
    for l, mode in enumerate(wl.modes):
        li = workloads.layer_inputs(wl, l)
        layers.append(dict(mode=mode, qI=li["qI"][b, q0:q0 + qn].float().numpy(), w=li["w"][b, q0:q0 + qn].numpy(),
                           q=li["q"][b, q0:q0 + qn].float().numpy(), swa=li["swa"][b, w0:w1].float().numpy()))
    need = set(wl.new_rows)
    for L in layers:
        if L["mode"] in (group.FULL, group.REINDEX):
            for i in range(qn):
                s = indexer.index_scores(L["qI"][i], L["w"][i], kI, int(n_vis[i]))
                need.update(int(p) for p in indexer.topk(s, wl.K)[0] if p >= 0)
    rows = np.array(sorted(need))
    kv = np.zeros((wl.N, 288), dtype=np.uint8)
    kv[rows] = fp4.quantize_kv_fp4(x[rows])
    new = x[wl.N - wl.n_new:].copy()
    return dict(kv=kv, kI=kI, layers=layers, new=new, n_vis=n_vis, queries=qn)


def oracle_row_step(wl, S):
    from oracle import group
    kv = S["kv"].copy()
    return group.group_row(kv, S["kI"], S["n_vis"], S["layers"], K=wl.K, W=wl.W,
                           swa_step=wl.swa_step, hsi_blocks=wl.hsi_blocks, hsi_block=wl.hsi_block,
                           kv_new=S["new"], new_rows=wl.new_rows)


def oracle_sample_text(wl):
    q0, qn = oracle_query_sample(wl)
    if qn == wl.Q:
        return "all queries of the row"
    return f"queries {q0}..{q0 + qn - 1} of the row's {wl.Q} (longest visible prefixes)"


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return 1


def cpu_baseline(wl):
    S = oracle_row_setup(wl, 0)
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_row_step(wl, S)
        n += 1
        if time.perf_counter() - t0 > 10.0:
            break
    dt = time.perf_counter() - t0
    return {"value": n * S["queries"] / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"batch row 0 of {wl.name}, {oracle_sample_text(wl)}, through the oracle's full group "
                      f"step ({len(wl.modes)} layers, quantise + scan + top-K + attention), {n} repetition(s), "
                      f"{dt:.1f} s; host os.cpu_count()={os.cpu_count()}"}


def run_reference(args, world, rank):
    wl = workloads.WORKLOADS[args.workload]
    if rank != 0:
        return
    setups = [oracle_row_setup(wl, b) for b in range(wl.B)]
    for _ in range(args.warmup):
        oracle_row_step(wl, setups[0])
    times = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        for S in setups:
            oracle_row_step(wl, S)
        times.append(time.perf_counter() - t0)
    mean = sum(times) / len(times)
    value = sum(S["queries"] for S in setups) / mean
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "Q": wl.Q, "N_entries": wl.N,
                       "layers": ",".join(workloads.MODE_NAMES[m] for m in wl.modes), "K": wl.K, "W": wl.W,
                       "parallelism": "oracle on host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"every batch row of {wl.name} per step, {oracle_sample_text(wl)}, "
                                       f"through the oracle group schedule (numpy, float64); warm-up steps "
                                       f"used row 0 only"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, world, rank, local):
    if rank == 0:
        _build.build()
    barrier(world)
    from fp4_kv_cache_mxfp4_b200 import csa2
    csa2.load()
    wl = workloads.WORKLOADS[args.workload]
    T = make_device_workload(wl, csa2, seed_shift=rank)
    st = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def eager_step():
        csa2.csa2_group_decode(T["g"], T["ws"])

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        flush.zero_()
        eager_step()
    torch.cuda.synchronize()
    st_code = csa2.csa2_device_status()
    if st_code != (0, 0):
        raise RuntimeError(f"device status after warm-up: {st_code}")
    # the step's launches (memset, quantise, scans, selections, attention)
    # replayed as one CUDA graph
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        eager_step()
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(graph):
        eager_step()
    torch.cuda.synchronize()
    step = graph.replay
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    # ---- timed: device-resident inputs
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for a, b in ev:
        flush.zero_()
        a.record(st)
        step()
        b.record(st)
    torch.cuda.synchronize()
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    mean_ms = max_over_ranks(sum(step_ms) / len(step_ms), world)

    # ---- traced pass: per-kernel durations with events on the launch stream
    launches_per_step = None
    csa2.csa2_trace_begin(64 * args.steps)
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for a, b in ev2:
        flush.zero_()
        a.record(st)
        eager_step()
        b.record(st)
    torch.cuda.synchronize()
    barrier(world)
    csa2.csa2_trace_stop()
    recs = csa2.csa2_trace_records()
    csa2.csa2_trace_end()
    traced_ms = sum(a.elapsed_time(b) for a, b in ev2) / args.steps
    launches_per_step = len(recs) / args.steps
    per_kernel = {}
    for name, ms in recs:
        c, t = per_kernel.get(name, (0, 0.0))
        per_kernel[name] = (c + 1, t + ms)

    # ---- end to end: host inputs -> device -> csa2_group_decode -> host outputs
    host_in = [(T["new"], torch.empty_like(T["new"], device="cpu").pin_memory())]
    for L in T["layers"]:
        for k in ("qI", "w", "q"):
            host_in.append((L[k], torch.empty_like(L[k], device="cpu").pin_memory()))
    for dev_t, host_t in host_in:
        host_t.copy_(dev_t)
    host_out = [(L["out"], torch.empty_like(L["out"], device="cpu").pin_memory()) for L in T["layers"]]
    h2d = sum(h.numel() * h.element_size() for _, h in host_in)
    d2h = sum(h.numel() * h.element_size() for _, h in host_out)
    ev3 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for a, b in ev3:
        flush.zero_()
        a.record(st)
        for dev_t, host_t in host_in:
            dev_t.copy_(host_t, non_blocking=True)
        step()
        for dev_t, host_t in host_out:
            host_t.copy_(dev_t, non_blocking=True)
        b.record(st)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev3) / args.steps, world)
    clk = clocks.stop()
    st_code = csa2.csa2_device_status()
    if st_code != (0, 0):
        raise RuntimeError(f"device status after the timed loops: {st_code}")

    if rank != 0:
        return
    queries = wl.B * wl.Q * world
    value = aggregate_queries_per_s(wl.B * wl.Q, world, mean_ms)
    peak, peak_kind = hbm_peak()
    n_scan, t_scan = per_kernel.get("index_scan_kernel", (0, 0.0))
    scan_ms = t_scan / max(n_scan, 1)
    scan_bytes = scan_algorithmic_bytes(wl)
    achieved = scan_bytes / (scan_ms * 1e-3) / 1e9 if n_scan else None
    if wl.prefill:
        # eight queries per MMA group make the prefill scan a contraction
        scan_flops = scan_algorithmic_flops(wl)
        t_peak, t_kind = tensor_peak()
        t_achieved = scan_flops / (scan_ms * 1e-3) / 1e12 if n_scan else None
        roofline = {"kernel": "index_scan_kernel", "bound": "tensor", "achieved": t_achieved, "peak": t_peak,
                    "peak_source": f"{t_kind} (MEASURED_PEAKS.json bf16_tflops_sustained)" if t_kind == "measured"
                    else "fallback 1.4 PFLOP/s sustained", "unit": "TFLOP/s",
                    "frac": (t_achieved / t_peak) if t_achieved else None, "traffic": None,
                    "algorithmic_flops_per_launch": scan_flops, "ms_per_launch": scan_ms, "launches": n_scan}
    sha = kernel_source_sha()
    traffic = SCAN_TRAFFIC["bytes_per_launch"] if (SCAN_TRAFFIC["sha"] == sha and args.workload == 2) else None
    step_bytes = step_algorithmic_bytes(wl)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": mean_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) caches and inputs)",
        "config": {"workload": wl.name, "B": wl.B, "Q": wl.Q, "N_entries": wl.N, "r": wl.r,
                   "layers": ",".join(workloads.MODE_NAMES[m] for m in wl.modes), "K": wl.K, "W": wl.W,
                   "kv_cache": "FP4 E2M1 + E4M3/16ch (288 B/entry)", "index_k": "bf16",
                   "l2": "flushed between steps (256 MB memset outside the timed events)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "hbm_gbs_step": step_bytes / (mean_ms * 1e-3) / 1e9,
        "hbm_frac_step": step_bytes / (mean_ms * 1e-3) / 1e9 / peak,
        "roofline": roofline if wl.prefill else
                    {"kernel": "index_scan_kernel", "bound": "hbm", "achieved": achieved, "peak": peak,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback 6.65 TB/s", "unit": "GB/s",
                     "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                     "algorithmic_bytes_per_launch": scan_bytes, "ms_per_launch": scan_ms,
                     "launches": n_scan},
        "kernels": {k: {"launches": c, "ms_mean": t / c} for k, (c, t) in sorted(per_kernel.items())},
        "ms_per_step_eager_traced": traced_ms,
        "launch": "CUDA graph of one csa2_group_decode call per step",
        "e2e": {"value": queries / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": int(round(launches_per_step * args.steps)) if launches_per_step else 0,
        "clocks": clk,
    }
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(wl)
    else:
        line["cpu_baseline"] = None
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
