"""GPU parity of tpla_cache_append (a new token's latent, optionally
Hadamard-rotated, RMS-normalised per shard, stored in the paged or contiguous
cache) against the float64 oracle, through the C ABI.

The kernel computes in f32 and rounds once to bf16; the oracle's float64 row
rounded to bf16 (round-to-nearest-even) is the reference.  The two differ
where the f32 value lies within rounding distance of a bf16 midpoint (one
bf16 step: relative 2^-7 bounds it), and, for the rare entries that the
Hadamard sums cancel to nearly zero, by the f32 rounding of those sums
itself: about 1e-6 on rows of unit RMS (a float32 restatement of the
transform shows 7e-7), which the absolute floor 2^-16 covers.  Almost all
stored values are equal.  Rows not written must be bit-identical to the
cache before the call."""

import numpy as np
import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from mla_latent_kv_dim_b200.workloads import as_f64, make_inputs
from oracle import tpla_oracle as O
from parity import assert_lse_close, assert_out_close, to_np

pytestmark = pytest.mark.gpu

POSITIONS = [0, 63, 64, 127, 300, 5, 191]


def _case(paged, in_dtype, seed):
    g = torch.Generator().manual_seed(seed)
    B = len(POSITIONS)
    pages = 5
    new = torch.randn((B, 576), generator=g) * torch.exp(-torch.arange(576) / 200.0) * 3.0
    new = new.to(in_dtype)
    if paged:
        nblk = B * pages + 3
        cache = torch.randn((nblk, 64, 576), generator=g).to(torch.bfloat16)
        pt = torch.randperm(nblk, generator=g)[: B * pages].reshape(B, pages).to(torch.int32)
    else:
        cache = torch.randn((B, 64 * pages, 576), generator=g).to(torch.bfloat16)
        pt = None
    return new, torch.tensor(POSITIONS, dtype=torch.int32), pt, cache


def _check_rows(got, before, want16, written):
    """got/before: bf16 cache tensors (CPU); want16: oracle cache rounded to
    bf16; written: boolean mask over rows [..., 576] that the call stores."""
    g = got.float().numpy()
    b = before.float().numpy()
    w = want16.float().numpy()
    untouched = ~written
    assert np.array_equal(g[untouched], b[untouched]), "rows outside the positions changed"
    gw, ww = g[written], w[written]
    err = np.abs(gw - ww)
    assert np.all(err <= 2.0 ** -7 * np.abs(ww) + 2.0 ** -16), f"max err {err.max()}"
    assert np.mean(gw == ww) >= 0.99


@pytest.mark.parametrize("groups,hadamard,in_dtype,paged", [
    (1, False, torch.float32, True), (1, True, torch.bfloat16, True),
    (2, True, torch.float32, True), (4, False, torch.bfloat16, False),
    (8, True, torch.float32, True), (2, False, torch.bfloat16, False)])
def test_cache_append_matches_oracle(cuda_dev, groups, hadamard, in_dtype, paged):
    new, pos, pt, cache = _case(paged, in_dtype, seed=groups * 10 + hadamard)
    eps = 1e-6
    d_cache = cache.to(cuda_dev)
    tp.cache_append(new.to(cuda_dev), pos.to(cuda_dev), None if pt is None else pt.to(cuda_dev),
                    d_cache, norm_groups=groups, hadamard=hadamard, eps=eps)
    torch.cuda.synchronize()
    assert tp.device_status() == 0
    want = O.cache_append_ref(as_f64(cache), as_f64(new), pos.numpy(),
                              None if pt is None else pt.numpy(), groups, hadamard, eps)
    want16 = torch.from_numpy(want).to(torch.bfloat16)
    written = np.zeros(cache.shape[:-1], dtype=bool)
    for b, p in enumerate(POSITIONS):
        if pt is None:
            written[b, p] = True
        else:
            written[pt[b, p // 64], p % 64] = True
    _check_rows(d_cache.cpu(), cache, want16, written)


def test_cache_append_out_of_range_sets_status(cuda_dev):
    new, pos, pt, cache = _case(True, torch.bfloat16, seed=5)
    pos[2] = 64 * pt.shape[1]  # past the request's pages
    pt[4, POSITIONS[4] // 64] = cache.shape[0] + 7  # page id outside the cache
    d_cache = cache.to(cuda_dev)
    tp.cache_append(new.to(cuda_dev), pos.to(cuda_dev), pt.to(cuda_dev), d_cache, 2, True)
    assert tp.device_status() == -6
    assert tp.device_status() == 0
    ok = [b for b in range(len(POSITIONS)) if b not in (2, 4)]  # requests 2, 4 are not written
    want = O.cache_append_ref(as_f64(cache), as_f64(new)[ok], pos.numpy()[ok], pt.numpy()[ok], 2,
                              True, 1e-6)
    written = np.zeros(cache.shape[:-1], dtype=bool)
    for b in ok:
        p = int(pos[b])
        written[pt[b, p // 64], p % 64] = True
    _check_rows(d_cache.cpu(), cache, torch.from_numpy(want).to(torch.bfloat16), written)


def test_append_then_decode_matches_oracle(cuda_dev):
    """The cache-write step followed by the decode it feeds: append one new
    token per request (Hadamard, per-shard norm for G = 2), then TPLA G = 2
    decode over the grown cache against the oracle on the oracle's own
    appended rows (rounded to bf16 like the stored cache)."""
    lens = [300, 64, 1, 129]
    w = make_inputs(4, 128, lens, paged=True, decay=True, seed=17, spare_blocks=2)
    # request 1 (64 tokens) grows into a second page: give it a spare block
    used = {int(w.page_table[b, k]) for b, L in enumerate(lens) for k in range((L + 63) // 64)}
    w.page_table[1, 1] = min(set(range(w.cache.shape[0])) - used)
    g = torch.Generator().manual_seed(3)
    new = torch.randn((4, 576), generator=g)
    pos = torch.tensor(lens, dtype=torch.int32)
    cache = w.cache.to(cuda_dev)
    tp.cache_append(new.to(cuda_dev), pos.to(cuda_dev), w.page_table.to(cuda_dev), cache, 2, True)
    seq = (pos + 1).to(cuda_dev)
    out, lse = tp.decode(w.q.to(cuda_dev), cache, seq, w.page_table.to(cuda_dev), 2, "replicate",
                         w.scale)
    torch.cuda.synchronize()
    assert tp.device_status() == 0
    grown = O.cache_append_ref(as_f64(w.cache), as_f64(new), lens, w.page_table.numpy(), 2, True,
                               1e-6)
    grown16 = as_f64(torch.from_numpy(grown).to(torch.bfloat16))
    rows = O.gather_request_rows(grown16, [L + 1 for L in lens], w.page_table.numpy())
    ro, rl = O.tpla_decode_ref(as_f64(w.q), rows, 2, "replicate", np.float32(w.scale))
    assert_out_close(to_np(out), ro)
    assert_lse_close(to_np(lse), rl)
