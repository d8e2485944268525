"""Tensor-parallel TPLA bookkeeping on CPU: two and four gloo ranks each hold
one shard's partial product and the all-reduce after the V up-projection
sums them into the combined output.  The per-rank products come from the
float64 oracle (the kernels need a GPU); what is tested here is the slicing
and the collective."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mla_latent_kv_dim_b200.tensor_parallel import (all_reduce_partials, head_slice,
                                                    shard_columns)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs():
    rng = np.random.default_rng(7)
    B, H, L = 2, 4, 40
    q = rng.standard_normal((B, H, 576))
    rows = [rng.standard_normal((L, 576)) for _ in range(B)]
    W = 0.02 * rng.standard_normal((H, 512, 32))
    return q, rows, W


def _worker(rank, world, port, results):
    from oracle import tpla_oracle as O
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, rows, W = _inputs()
        out_g, _ = O.tpla_decode_ref(q, rows, world, "replicate", 0.1, shard=rank)
        cols = shard_columns(world, rank)
        y = torch.from_numpy(O.vup_ref(out_g, W[:, cols, :]))  # this rank's partial product
        all_reduce_partials(y)
        results[rank] = y.numpy()
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_all_reduce_of_partials_is_the_combined_output(world):
    from oracle import tpla_oracle as O
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), results), nprocs=world,
                       start_method="spawn", join=True)
    q, rows, W = _inputs()
    full, _ = O.tpla_decode_ref(q, rows, world, "replicate", 0.1)
    want = O.vup_ref(full, W)
    for r in range(world):
        np.testing.assert_allclose(results[r], want, rtol=1e-12, atol=1e-12)


def test_single_process_all_reduce_is_identity():
    y = torch.arange(6.0)
    assert all_reduce_partials(y) is y and y.tolist() == [0, 1, 2, 3, 4, 5]


def test_slices():
    assert shard_columns(1, 0) == slice(0, 512)
    assert shard_columns(2, 1) == slice(256, 512)
    assert shard_columns(4, 2) == slice(256, 384)
    assert head_slice(128, 2, 1) == slice(64, 128)
    for bad in ((3, 0), (2, 2), (2, -1)):
        with pytest.raises(ValueError):
            shard_columns(*bad)
    with pytest.raises(ValueError):
        head_slice(6, 4, 0)
