"""Rank logic of the multi-GPU benchmark, run as world-size-2 gloo process groups on CPU.

Every (batch, head) and every attention call is independent, so ranks share no data: the
only cross-rank steps are the barriers around the timed region and the max-over-ranks
reduction of the timings.
"""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 * (rank + 1) + 0.5
        dist.barrier()
        m = bench.max_over_ranks(local_ms, torch.device("cpu"))
        seed = bench.rank_seed(0, rank)
        out[rank] = (m, seed)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_seeds_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 20.5          # every rank sees the slowest rank's time
    assert out[0][1] != out[1][1]                  # independent problems per rank


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25


def test_aggregate_is_weak_scaling_sum():
    one = bench.aggregate_tflops(2.0e12, 10.0, 1)
    assert bench.aggregate_tflops(2.0e12, 10.0, 4) == pytest.approx(4 * one)
    assert one == pytest.approx(200.0)


def test_reference_arm_only_on_rank_zero(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 1, 3, 2
    bench.reference_arm(A(), bench.synthetic.TINY)
    assert capsys.readouterr().out == ""
