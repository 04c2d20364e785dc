"""The bench's multi-rank host logic (replicas, barrier, max over ranks,
whole-job throughput) on two CPU processes over gloo: no GPU involved."""

import os
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from fp4_kv_cache_mxfp4_b200 import workloads
    from fp4_kv_cache_mxfp4_b200.device_workload import with_seed_shift
    w, r, _ = bench.dist_setup(backend="gloo")
    try:
        bench.barrier(w)
        ms = 10.0 + 5.0 * r                          # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, w)
        wl = with_seed_shift(workloads.WORKLOADS[2], r)
        kI_first = float(workloads.index_k(wl, 0)[0, 0])
        value = bench.aggregate_queries_per_s(wl.B * wl.Q, w, worst)
        out.put((r, worst, wl.seed, (wl.B, wl.Q, wl.N), kI_first, value))
        bench.barrier(w)
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_replicas_and_max_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, worst0, seed0, shape0, k0, v0), (r1, worst1, seed1, shape1, k1, v1) = res
    assert worst0 == worst1 == 15.0                 # both ranks see the slowest rank's time
    assert seed0 != seed1 and shape0 == shape1       # replicas: same shapes, own inputs
    assert k0 != k1
    assert v0 == v1 == pytest.approx(4 * 2 / 15e-3)  # all ranks' queries over the slowest step
