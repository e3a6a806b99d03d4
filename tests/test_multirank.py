"""The multi-rank host path of bench.py on CPU with two gloo ranks: the
timing reduction (max over ranks), the barrier, the whole-job value, and the
reference arm's rank handling (rank 0 alone runs it)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist = bench.init_dist(world, "gloo")
    try:
        bench.barrier(dist)
        ms = 10.0 + 5.0 * rank                  # rank 1 is the slow one
        ms_max = bench.reduce_max(ms, dist)
        value = bench.whole_job_value(1e9, 4, world, ms_max)
        q.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_max, value in got:
        assert ms_max == 15.0
        # 2 ranks x 4 steps x 1 GB in 15 ms
        assert value == pytest.approx(2 * 4 * 1e9 / 15e-3 / 1e9)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup, gpus = 1, 3, 2
    assert bench.run_reference(Args()) == 0      # returns at once, no work, no output


def test_whole_job_value_single_rank():
    assert bench.whole_job_value(179.8e6, 1000, 1, 457.3) == pytest.approx(393.2, rel=1e-3)
