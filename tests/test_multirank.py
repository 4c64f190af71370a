"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

The attention path needs no collective (every (b, h) is an independent
problem); the only cross-rank steps are the barrier and the max-over-ranks of
the device timings, which these tests exercise without a GPU."""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank 1 is the slow one: every rank must see its time
        local_ms = 10.0 + 5.0 * rank
        got = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(3.5, None, None) == 3.5


def test_whole_job_value_is_weak_scaling():
    one = bench.whole_job_tflops(1, 2.0e12, 10, 20.0)
    assert one == pytest.approx(1000.0)
    assert bench.whole_job_tflops(4, 2.0e12, 10, 20.0) == pytest.approx(4 * one)
