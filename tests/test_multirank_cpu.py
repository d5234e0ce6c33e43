"""Replica plumbing of bench.py on CPU ranks (gloo, world size 2).

The codec has no exchange step, so `bench.py --gpus N` runs N replicas and
the only collective is the max-over-ranks reduction of the device time.
These tests run that reduction on two gloo ranks and check the whole-job
throughput formula (weak scaling).
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


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank)
        q.put((rank, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 15.0), (1, 15.0)]


def test_max_over_ranks_without_process_group_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_job_value_is_weak_scaling():
    one = bench.job_value(1, 1.0e9, 1.0)
    assert one == pytest.approx(1000.0)
    assert bench.job_value(4, 1.0e9, 1.0) == pytest.approx(4 * one)
