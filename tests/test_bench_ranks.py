"""Host logic of the multi-process bench (one process per GPU, replicas of the step):
max-over-ranks timing, whole-job throughput, and rank 0 alone printing the reference arm.
Run with the gloo backend on CPU, world size 2."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(times[rank], device="cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    world, port = 2, _free_port()
    times = [3.5, 7.25]
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert dict(out) == {0: 7.25, 1: 7.25}


def test_single_process_time_is_unchanged():
    assert bench.max_over_ranks(4.0) == 4.0


def test_job_throughput_is_weak_scaling_aggregate():
    # 1 GB per step per rank, 10 steps, 2 ranks, 1 s on the slowest rank -> 20 GB/s
    assert bench.job_throughput(10**9, 10, 2, 1000.0) == pytest.approx(20.0)
    assert bench.job_throughput(10**9, 10, 1, 1000.0) == pytest.approx(10.0)


def test_reference_arm_prints_on_rank_0_only(monkeypatch, capsys):
    class Args:
        gpus, steps, warmup = 2, 3, 3

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(Args) == 0
    assert capsys.readouterr().out == ""


def test_dist_env_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)
    monkeypatch.setenv("RANK", "3")
    monkeypatch.setenv("WORLD_SIZE", "8")
    monkeypatch.setenv("LOCAL_RANK", "3")
    assert bench.dist_env() == (3, 8, 3)
