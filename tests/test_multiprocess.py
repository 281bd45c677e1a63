"""Multi-rank plumbing of bench.py on the host: two gloo ranks on CPU.

The path has no data-path collective (replicas only): each rank runs the whole step on its
own GPU, the timed region is bracketed by barriers and the slowest rank's time sets the
whole-job throughput.  These tests run that plumbing with world size 2 over gloo: the max
over ranks, the barrier, the throughput aggregation and the reference arm, which only
rank 0 runs.
"""
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        bench = _load_bench()
        bench.barrier(ws)
        # per-rank elapsed times: rank 1 is the slow one
        mine = [12.5, 30.25][rank]
        slowest = bench.max_over_ranks(mine, ws)
        bench.barrier(ws)
        value = bench.replica_throughput(ws, 1.0e9, 4, slowest)

        class Args:
            workload = "720p-small"
            warmup = 0
            steps = 0
            gpus = ws
        # the reference arm: rank 0 alone works; the others return at once without output
        ref_rc = bench.run_reference(Args, ws, rank) if rank != 0 else None
        out.put((rank, slowest, value, ref_rc))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in results] == [0, 1]
    for rank, slowest, value, ref_rc in results:
        assert slowest == pytest.approx(30.25)
        # 2 replicas x 1e9 units x 4 steps in 30.25 ms
        assert value == pytest.approx(2 * 1.0e9 * 4 / 0.03025)
    assert results[1][3] == 0          # rank 1 of the reference arm exits 0 without work


def test_single_rank_needs_no_process_group():
    bench = _load_bench()
    assert bench.max_over_ranks(7.0, 1) == 7.0
    bench.barrier(1)
    assert bench.replica_throughput(1, 10.0, 2, 1000.0) == pytest.approx(20.0)
