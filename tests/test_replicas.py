"""Replica timing bookkeeping on CPU: two gloo ranks, each with its own time;
the job's time is the slowest rank's and the rate aggregates all ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mla_latent_kv_dim_b200.replicas import aggregate_rate, max_over_ranks


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [10.0 + 5.0 * rank, 2.0 - rank]  # rank 1 slower on the first, faster on the second
        got = max_over_ranks(ms, dist, torch.device("cpu"))
        rate, t_step = aggregate_rate(world, 1000.0, got[0], 5)
        results[rank] = (got, rate, t_step)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), results), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        got, rate, t_step = results[r]
        assert got == [15.0, 2.0]                    # element-wise max over ranks
        assert t_step == pytest.approx(15.0 / 1e3 / 5)
        assert rate == pytest.approx(2 * 1000.0 / t_step)


def test_single_process_is_identity():
    assert max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    rate, t = aggregate_rate(1, 64.0, 20.0, 10)
    assert t == pytest.approx(2e-3) and rate == pytest.approx(32000.0)
    with pytest.raises(ValueError):
        aggregate_rate(1, 1.0, 0.0, 10)
