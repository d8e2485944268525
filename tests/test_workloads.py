"""The seeded input recipe: the named workloads have the shapes, length
mixes, paging and value distributions of the configurations they stand in
for (DeepSeek-V2-Lite, DeepSeek-V3, Kimi-K2 and long-context shapes), and the
generator is deterministic per seed.  CPU only."""

import math

import numpy as np
import pytest
import torch

from mla_latent_kv_dim_b200.workloads import CONFIGS, SOFTMAX_SCALE, make_inputs, make_workload

SPEC = {  # name: B, H, lengths, paged, channel decay, seed, W_uv
    "tiny": (1, 16, ("fixed", 256), False, False, 0, False),
    "v2lite": (32, 16, ("uniform", 2048, 4096), True, True, 1, True),
    "dsv3": (64, 128, ("fixed", 32768), True, True, 2, True),
    "kimi": (16, 64, ("uniform", 16384, 32768), True, True, 3, True),
    "long": (4, 128, ("fixed", 131072), True, True, 4, False),
}


@pytest.mark.parametrize("name", sorted(SPEC))
def test_named_configs(name):
    B, H, lens, paged, decay, seed, wuv = SPEC[name]
    c = CONFIGS[name]
    assert (c["B"], c["H"], c["lens"], c["paged"], c["decay"], c["seed"], c["wuv"]) == \
        (B, H, lens, paged, decay, seed, wuv)


def test_softmax_scale_is_one_over_sqrt_192():
    assert SOFTMAX_SCALE == 1.0 / math.sqrt(128 + 64)


@pytest.mark.parametrize("name", ["tiny", "v2lite", "kimi"])
def test_generated_shapes_and_lengths(name):
    B, H, lens, paged, decay, seed, wuv = SPEC[name]
    w = make_workload(name)
    assert w.q.shape == (B, H, 576) and w.q.dtype == torch.bfloat16
    L = w.seq_lens.numpy()
    assert w.seq_lens.dtype == torch.int32 and L.shape == (B,)
    if lens[0] == "fixed":
        assert np.all(L == lens[1])
    else:
        assert L.min() >= lens[1] and L.max() <= lens[2]
        assert len(set(L.tolist())) > B // 2  # a mix of lengths, not one value
    if paged:
        assert w.cache.shape[1:] == (64, 576) and w.cache.dtype == torch.bfloat16
        pt = w.page_table.numpy()
        used = np.concatenate([pt[b, :(int(L[b]) + 63) // 64] for b in range(B)])
        # every page of every request is its own physical block
        assert len(np.unique(used)) == len(used)
        assert used.min() >= 0 and used.max() < w.cache.shape[0]
        # random physical order, not the identity
        assert not np.array_equal(used, np.arange(len(used)))
    else:
        assert w.page_table is None and w.cache.shape == (B, int(L.max()), 576)
    if wuv:
        assert w.W_uv.shape == (H, 512, 128) and w.W_uv.dtype == torch.bfloat16
        assert abs(w.W_uv.float().std().item() - 0.02) < 0.001
    else:
        assert w.W_uv is None


def test_deterministic_per_seed():
    a = make_inputs(3, 8, ("uniform", 10, 300), paged=True, decay=True, seed=11, wuv=True)
    b = make_inputs(3, 8, ("uniform", 10, 300), paged=True, decay=True, seed=11, wuv=True)
    c = make_inputs(3, 8, ("uniform", 10, 300), paged=True, decay=True, seed=12, wuv=True)
    for x, y in ((a.q, b.q), (a.cache, b.cache), (a.page_table, b.page_table),
                 (a.seq_lens, b.seq_lens), (a.W_uv, b.W_uv)):
        assert torch.equal(x, y)
    assert not torch.equal(a.q, c.q)


def test_channel_decay_and_distributions():
    """Latent channel j has standard deviation exp(-j/128) (log-std slope
    -1/128 fitted over the 512 channels); rope channels and q are N(0, 1)."""
    w = make_inputs(8, 16, ("fixed", 4096), paged=True, decay=True, seed=13)
    rows = w.cache.float().reshape(-1, 576).numpy().astype(np.float64)
    sd = rows.std(axis=0)
    slope, icpt = np.polyfit(np.arange(512), np.log(sd[:512]), 1)
    assert abs(slope + 1 / 128) < 2e-4 and abs(icpt) < 0.02
    assert np.all(np.abs(sd[512:] - 1.0) < 0.02)
    assert abs(rows.mean()) < 0.01
    qv = w.q.float().numpy()
    assert abs(qv.std() - 1.0) < 0.02 and abs(qv.mean()) < 0.02
    flat = make_inputs(2, 4, ("fixed", 4096), paged=True, decay=False, seed=13)
    sd0 = flat.cache.float().reshape(-1, 576).numpy().std(axis=0)
    assert np.all(np.abs(sd0 - 1.0) < 0.03)
