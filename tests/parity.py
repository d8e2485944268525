"""Shared comparison helpers for the GPU parity tests (no method arithmetic).

Tolerance (bf16 inputs, f32 accumulation):
  outputs: max|got - ref| <= 1e-2 * max|ref|  and
           mean|got - ref| / mean|ref| <= 2e-3;
  lse:     |got - ref| <= 1e-2 absolute where finite; -inf must match.
End-to-end checks through a bf16 re-rounding (Hadamard) use ``factor`` 2.
"""
from __future__ import annotations

import numpy as np
import torch

from mla_latent_kv_dim_b200.workloads import Workload, as_f64
from oracle import tpla_oracle as O

MAX_REL = 1e-2
MEAN_REL = 2e-3
LSE_ABS = 1e-2


def assert_out_close(got, ref, factor: float = 1.0, what: str = "out"):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    scale = np.abs(ref).max()
    if scale == 0:
        assert err.max() == 0, what
        return
    assert err.max() <= factor * MAX_REL * scale, (
        f"{what}: max err {err.max():.3e} > {factor * MAX_REL:.0e} * {scale:.3e}")
    mean_rel = err.mean() / np.abs(ref).mean()
    assert mean_rel <= factor * MEAN_REL, f"{what}: mean rel err {mean_rel:.3e}"


def assert_lse_close(got, ref, factor: float = 1.0, what: str = "lse"):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), f"{what}: -inf pattern differs"
    if fin.any():
        err = np.abs(got[fin] - ref[fin]).max()
        assert err <= factor * LSE_ABS, f"{what}: max abs err {err:.3e}"


def to_device(w: Workload, dev):
    return dict(q=w.q.to(dev), cache=w.cache.to(dev), seq_lens=w.seq_lens.to(dev),
                page_table=None if w.page_table is None else w.page_table.to(dev))


def oracle_rows(w: Workload, requests=None):
    """float64 cache rows of the chosen requests (all by default)."""
    reqs = range(w.B) if requests is None else requests
    cache = w.cache
    rows = []
    for b in reqs:
        L = int(w.seq_lens[b])
        if w.page_table is None:
            rows.append(as_f64(cache[b, :L]))
        else:
            pages = (L + 63) // 64
            blk = w.page_table[b, :pages].long()
            r = cache[blk].reshape(pages * 64, cache.shape[-1])[:L]
            rows.append(as_f64(r))
    return rows


def oracle_decode(w: Workload, G, rope_mode, shard=None, requests=None, q=None, rows=None):
    reqs = list(range(w.B)) if requests is None else list(requests)
    qf = as_f64(w.q if q is None else q)[reqs]
    rows = oracle_rows(w, reqs) if rows is None else rows
    return O.tpla_decode_ref(qf, rows, G, rope_mode, np.float32(w.scale), shard)


def to_np(t: torch.Tensor):
    return t.detach().float().cpu().numpy().astype(np.float64)
