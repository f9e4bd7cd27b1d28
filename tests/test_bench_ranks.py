"""The replica (N > 1) host path of bench.py, on CPU with the gloo backend.

Each rank runs an independent stack; the step time is the slowest rank's
(an all-reduce MAX), the value counts every rank's tokens, and the reference
arm runs on rank 0 only.
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")  # ranks take 10 and 15 ms
        value = bench.job_value(128, world, ms)
        dist.barrier()
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        ms, value = out[rank]
        assert ms == 15.0                            # the slowest rank
        assert value == pytest.approx(2 * 128 / 0.015)  # all ranks' tokens


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5
    assert bench.job_value(64, 1, 8.0) == pytest.approx(8000.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:  # would fail at once if rank 1 touched any of it
        pass
    assert bench.run_reference(Args(), 1, 2, 1) is None
    assert capsys.readouterr().out == ""
