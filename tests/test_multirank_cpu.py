"""The N > 1 host path of bench.py on CPU: world_size 2 over gloo.

The path shards as independent replicas (no data-path collective): each rank
times its own sweep, the ranks meet at a barrier on both sides of the timed
region, the slowest rank's time is taken, and the whole-job value counts
every rank's bytes.  The reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(world, times[rank])
        bench.barrier(world)
        value = bench.whole_job_gbs(world, bench.step_weight_bytes(), 100, ms)
        out.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_bytes():
    world, times = 2, [3.25, 4.5]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    expect = world * bench.step_weight_bytes() * 100 / (max(times) * 1e-3) / 1e9
    for rank, ms, value in got:
        assert ms == max(times)
        assert value == pytest.approx(expect, rel=1e-12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(1, 2.5) == 2.5
    bench.barrier(1)
    assert bench.whole_job_gbs(1, 1e9, 10, 1000.0) == pytest.approx(10.0)


def test_reference_arm_runs_on_rank_zero_only():
    class A:
        steps, warmup, gpus = 1, 3, 2
    assert bench.run_reference(A(), 2, 1) is None
