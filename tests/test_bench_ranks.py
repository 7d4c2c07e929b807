"""Multi-rank logic of bench.py on CPU: two gloo ranks take the barrier, agree
on the max of their timed regions, and the whole-job throughput counts every
rank's tokens over the slowest rank's time.  The reference arm does its work
on rank 0 only."""
import datetime
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, _ = bench.dist_env()
        bench.barrier(w)
        ms = 10.0 + 5.0 * r  # this rank's timed region
        ms_max = bench.max_over_ranks(ms, w, torch)
        bench.barrier(w)
        q.put((r, w, ms_max, bench.job_throughput(w, 100, 4, ms_max)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort()
    assert [g[0] for g in got] == [0, 1]
    for _, w, ms_max, value in got:
        assert w == 2
        assert ms_max == 15.0  # the slower rank's time
        assert value == 2 * 100 * 4 / 15.0e-3


def test_job_throughput_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_throughput(1, 1000, 1, 75.0) == 1000 / 75.0e-3


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import argparse
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(config=1, steps=1, warmup=1, gpus=2, impl="reference")
    assert bench.run_reference(args) == 0  # returns before any oracle work
