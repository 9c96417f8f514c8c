"""Rank coordination of the benchmark on CPU: two gloo ranks (world size 2).

The path shards into independent replicas (no data-path collective), so the
only multi-rank logic is the host side of bench.py: every timed quantity is
the slowest rank's (a MAX all-reduce), the job rate is the per-rank work times
the world size over that time, and under torchrun only rank 0 runs and prints
the reference arm."""
import datetime
import os
import socket
import types

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports 1 + 2.5 r ms: both must see the slowest rank's time
        t = bench.max_over_ranks(1.0 + 2.5 * rank, dist)
        dist.barrier()
        rate = bench.job_rate(2.0e12, world, t * 1e-3)
        out.put((rank, t, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in procs:
            rank, t, rate = out.get(timeout=120)
            res[rank] = (t, rate)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    assert res[0] == res[1]
    t, rate = res[0]
    assert t == pytest.approx(3.5)
    assert rate == pytest.approx(2.0 * 2.0e12 / 3.5e-3)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(4.25, None) == 4.25
    assert bench.job_rate(10.0, 1, 5.0) == 2.0
    assert bench.job_rate(10.0, 4, 5.0) == 8.0


def test_reference_arm_runs_on_rank_zero_only(capsys):
    args = types.SimpleNamespace(gpus=2, steps=1, warmup=0, cpu_rows=16)
    assert bench.run_reference(args, 1) is None
    assert capsys.readouterr().out == ""
