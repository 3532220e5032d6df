"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, the max over ranks of the
timings and the whole-job throughput (replicas: each rank runs its own call)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured (10 + r, 2 - r) ms: the job time is the slowest rank's
        got = bench.max_over_ranks([10.0 + rank, 2.0 - rank], torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0] == out[1] == [11.0, 2.0]


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench

    one = bench.job_throughput(4e12, 1, 10.0)
    assert one == pytest.approx(400.0)
    assert bench.job_throughput(4e12, 8, 10.0) == pytest.approx(8 * one)


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]
