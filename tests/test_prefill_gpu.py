"""GPU parity of tpla_prefill (prompt rows into the paged cache, then exact
MLA of every prompt token over its causal prefix) against the float64
oracle, through the C ABI; and prefill followed by TPLA decode over the
rows it stored.

The oracle side stores the rows with ``cache_append_ref``, rounds the cache
to bf16 as the GPU stores it, and runs ``mla_prefill_ref`` over the
request's rows.  Tolerances are the decode parity tests' (bf16 inputs, f32
accumulation)."""

import numpy as np
import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from mla_latent_kv_dim_b200.workloads import as_f64, make_prefill_inputs
from oracle import tpla_oracle as O
from parity import assert_lse_close, assert_out_close, to_np

pytestmark = pytest.mark.gpu


def _oracle(w, groups, hadamard, rows_idx=None, eps=1e-6):
    T = w.q.shape[0]
    pos = w.start + np.arange(T)
    grown = O.cache_append_ref(as_f64(w.cache), as_f64(w.kv_new), pos,
                               np.tile(w.page_row.numpy(), (T, 1)), groups, hadamard, eps)
    grown16 = torch.from_numpy(grown).to(torch.bfloat16)
    rows = O.gather_request_rows(as_f64(grown16), [w.start + T], w.page_row.numpy()[None])[0]
    q = as_f64(w.q)
    if rows_idx is None:
        out, lse = O.mla_prefill_ref(q, rows, w.start, np.float32(w.scale))
        return grown16, out, lse
    # sampled prompt tokens: token i is the prefill of a prompt that ends at i
    outs, lses = [], []
    for i in rows_idx:
        o, l = O.mla_prefill_ref(q[i:i + 1], rows[:w.start + i + 1], w.start + i,
                                 np.float32(w.scale))
        outs.append(o[0])
        lses.append(l[0])
    return grown16, np.stack(outs), np.stack(lses)


def _run(w, dev, groups, hadamard, out_dtype=torch.float32):
    cache = w.cache.to(dev)
    out, lse = tp.prefill(w.q.to(dev), w.kv_new.to(dev), w.start, w.page_row.to(dev), cache,
                          norm_groups=groups, hadamard=hadamard, scale=w.scale,
                          out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert tp.device_status() == 0
    return cache, out, lse


@pytest.mark.parametrize("T,H,start,groups,hadamard,out_dtype", [
    (300, 128, 0, 1, False, torch.float32),    # several 256-token tiles, ragged tail
    (77, 16, 130, 2, True, torch.bfloat16),     # chunked: a cached prefix, small H
    (1, 64, 0, 1, False, torch.float32),        # one token: its own row only
    (64, 256, 191, 4, True, torch.float32),     # two 128-head groups
])
def test_prefill_matches_oracle(cuda_dev, T, H, start, groups, hadamard, out_dtype):
    w = make_prefill_inputs(T, H, start, seed=T + H + start)
    cache, out, lse = _run(w, cuda_dev, groups, hadamard, out_dtype)
    grown16, ro, rl = _oracle(w, groups, hadamard)
    # stored rows: the oracle's rounded rows within one bf16 step, plus the
    # f32 rounding of the Hadamard sums where they cancel to nearly zero
    # (the bound of the cache-append parity test)
    got = cache.cpu().float().numpy()
    want = grown16.float().numpy()
    assert np.all(np.abs(got - want) <= 2.0 ** -7 * np.abs(want) + 2.0 ** -16)
    assert np.mean(got == want) >= 0.99
    assert_out_close(to_np(out), ro)
    assert_lse_close(to_np(lse)[:, :, 0], rl)


def test_prefill_launches_append_decode_merge(cuda_dev):
    w = make_prefill_inputs(40, 128, 0, seed=5)
    torch.cuda.synchronize()
    before = tp.launch_count()
    _run(w, cuda_dev, 1, False)
    # the cache write, the tcgen05 attention kernel and the split-KV merge
    assert tp.launch_count() - before == 3


def test_prefill_then_tpla_decode(cuda_dev):
    """Prefill/decode separation: exact MLA over the prompt, then one TPLA
    G=2 decode step of the request over the rows the prefill stored plus the
    new token's row."""
    T, H = 200, 128
    w = make_prefill_inputs(T, H, 0, seed=11)
    cache, out, lse = _run(w, cuda_dev, 2, True)
    g = torch.Generator().manual_seed(12)
    qd = torch.randn((1, H, 576), generator=g).to(torch.bfloat16)
    new = torch.randn((1, 576), generator=g)
    pos = torch.tensor([T], dtype=torch.int32)
    pt = w.page_row[None].contiguous()
    tp.cache_append(new.to(cuda_dev), pos.to(cuda_dev), pt.to(cuda_dev), cache, 2, True)
    dout, dlse = tp.decode(qd.to(cuda_dev), cache, (pos + 1).to(cuda_dev), pt.to(cuda_dev), 2,
                           "replicate", w.scale)
    torch.cuda.synchronize()
    assert tp.device_status() == 0
    grown16, ro, rl = _oracle(w, 2, True)
    assert_out_close(to_np(out), ro)
    assert_lse_close(to_np(lse)[:, :, 0], rl)
    after = O.cache_append_ref(as_f64(grown16), as_f64(new), [T], pt.numpy(), 2, True, 1e-6)
    after16 = as_f64(torch.from_numpy(after).to(torch.bfloat16))
    rows = O.gather_request_rows(after16, [T + 1], pt.numpy())
    do, dl = O.tpla_decode_ref(as_f64(qd), rows, 2, "replicate", np.float32(w.scale))
    assert_out_close(to_np(dout), do)
    assert_lse_close(to_np(dlse), dl)


@pytest.mark.slow
def test_prefill_dsv3_prompt_sampled(cuda_dev):
    """A 4096-token DeepSeek-V3-shaped prompt (H = 128) in the launch
    configuration the benchmark times; sampled prompt tokens against the
    oracle (tile edges, the first and the last token)."""
    T, H = 4096, 128
    w = make_prefill_inputs(T, H, 0, seed=21)
    cache, out, lse = _run(w, cuda_dev, 1, False)
    idx = [0, 1, 255, 256, 1000, 2047, 4095]
    grown16, ro, rl = _oracle(w, 1, False, rows_idx=idx)
    o = to_np(out)[idx]
    assert_out_close(o, ro)
    assert_lse_close(to_np(lse)[idx, :, 0], rl)
