"""The benchmark's algorithmic byte and FLOP counts, checked against the
per-token figures written out by hand from the cache layout (576 bf16 values
per token: 512 latent + 64 rope) and the shard definitions."""
import os
import sys

import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from mla_latent_kv_dim_b200.workloads import make_inputs  # noqa: E402


@pytest.fixture(scope="module")
def w():
    return make_inputs(3, 4, [100, 0, 64], paged=True, seed=5)


def test_full_mode_reads_every_value_once(w):
    # 164 tokens x 576 values x 2 bytes, independent of G (rope read once)
    for G in (1, 2, 4, 8):
        assert w.latent_kv_bytes(G) == 164 * 1152


@pytest.mark.parametrize("G,rope,per_tok", [(1, "replicate", 1152), (2, "replicate", 640),
                                            (4, "replicate", 384), (2, "split", 576),
                                            (4, "split", 288)])
def test_one_shard_bytes(w, G, rope, per_tok):
    # one rank's share: its 512/G latent columns plus all (replicate) or
    # 64/G (split) rope columns; 640 = 2 x 320 is the pages' TP=2 width
    assert w.latent_kv_bytes(G, shard=0, rope_mode=rope) == 164 * per_tok


@pytest.mark.parametrize("G,shard,rope,flops", [
    (1, None, "replicate", 2 * 576 + 2 * 512),            # exact MLA: 2176
    (2, None, "replicate", 2 * (2 * 320 + 2 * 256)),      # 2304
    (4, None, "replicate", 4 * (2 * 192 + 2 * 128)),
    (2, None, "split", 2 * (2 * 288 + 2 * 256)),
    (2, 0, "replicate", 2 * 320 + 2 * 256),
    (4, 1, "split", 2 * 144 + 2 * 128),
])
def test_flops_per_token_head(G, shard, rope, flops):
    assert bench.flops_per_token_head(G, shard, rope) == flops


def test_benchmark_arithmetic_intensity():
    # the DeepSeek-V3 step (G=2, rope replicated): 2304 flops per token-head,
    # 1152 bytes per token, 128 heads -> 256 flops per byte
    assert bench.flops_per_token_head(2) * 128 / 1152 == 256


def test_one_shard_speedups_divide_g1_time_by_the_shard_time():
    vs_G = [{"G": 1, "mode": "full", "decode_us": 800.0},
            {"G": 2, "mode": "full", "decode_us": 810.0},
            {"G": 2, "mode": "one-shard", "decode_us": 400.0},
            {"G": 4, "mode": "one-shard", "decode_us": 320.0}]
    assert bench.one_shard_speedups(vs_G) == {"G2": 2.0, "G4": 2.5}
    assert bench.one_shard_speedups([]) is None
    assert bench.one_shard_speedups(vs_G[1:]) is None
