"""The multi-process side of bench.py on CPU: two gloo ranks (one process per rank, as
torchrun launches them) check the max-over-ranks timing and the whole-job throughput that
every N > 1 bench line uses; the reference arm runs on rank 0 only."""

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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 100.0 + 37.5 * rank                 # the ranks finish at different times
        slowest = bench.max_over_ranks(local_ms, world)
        dist.barrier()
        rate = bench.whole_job_rate(world, 2.0e12, 4, slowest)
        out[rank] = (slowest, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 137.5
    # every rank reports the same whole-job rate: 2 ranks x 4 steps x 2 TFLOP in 137.5 ms
    assert out[0][1] == out[1][1] == pytest.approx(2 * 4 * 2.0 / 0.1375)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.whole_job_rate(1, 1e12, 10, 1000.0) == pytest.approx(10.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class A:
        workload, warmup, steps = "tiny-1x1024-d64-fp32", 0, 1
    assert bench.run_reference(A(), world=2, rank=1) is None
    assert capsys.readouterr().out == ""
