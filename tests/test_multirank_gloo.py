"""The multi-process path of bench.py on CPU: two gloo ranks, each with its
own timings; the timing reduction must give every rank the maximum and the
whole-job rate must count the work of all ranks over the slowest rank."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local = [10.0 + 5.0 * rank, 3.0 - rank]           # rank 0: (10, 3), rank 1: (15, 2)
        got = bench.reduce_max_over_ranks(local, world, torch.device("cpu"))
        rate = bench.whole_job_rate(2.0, 4, world, got[0])
        out[rank] = got + [rate]
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_rate():
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork of this (possibly CUDA) process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        assert out[r][0] == 15.0 and out[r][1] == 3.0
        # 2 units/step x 4 steps x 2 ranks over 15 ms
        assert out[r][2] == pytest.approx(2.0 * 4 * 2 / 0.015)


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max_over_ranks([1.5, 2.0], 1, torch.device("cpu")) == [1.5, 2.0]
