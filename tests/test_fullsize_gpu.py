"""GPU parity at the full workload sizes (DeepSeek-V3, Kimi-K2, DeepSeek-V2-Lite
and long-context shapes), in the launch configuration the benchmark uses
(persistent balanced split-KV unless a test names explicit splits).

The float64 oracle cannot afford every request of the large shapes, so those
tests compare a few sampled requests, all heads and all tokens of each,
element by element; the small shape is compared whole.
"""

import numpy as np
import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from mla_latent_kv_dim_b200.workloads import make_workload
from oracle import tpla_oracle as O
from parity import as_f64, assert_lse_close, assert_out_close, oracle_rows, to_device, to_np

pytestmark = pytest.mark.gpu


def rotated_bf16(x, dim=512):
    """The oracle's own Hadamard rotation of bf16 values, rounded to bf16 like
    the stored rotated cache."""
    return as_f64(torch.from_numpy(O.hadamard_ref(as_f64(x), dim)).to(torch.bfloat16))


def decode(d, w, G, rope, num_splits=0):
    out, lse = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], G, rope, w.scale,
                         num_splits=num_splits)
    torch.cuda.synchronize()
    assert tp.device_status() == 0
    return to_np(out), to_np(lse)


def check_requests(w, out, lse, reqs, G, rope, q=None, rows=None):
    qf = as_f64(w.q)[reqs] if q is None else q
    rows = oracle_rows(w, reqs) if rows is None else rows
    ro, rl = O.tpla_decode_ref(qf, rows, G, rope, np.float32(w.scale))
    assert_out_close(out[reqs], ro)
    assert_lse_close(lse[reqs], rl)
    return ro


@pytest.fixture(scope="module")
def dsv3():
    return make_workload("dsv3")


def test_dsv3_mla_g1_sampled(cuda_dev, dsv3):
    w = dsv3
    d = to_device(w, cuda_dev)
    out, lse = decode(d, w, 1, "replicate")
    check_requests(w, out, lse, [0, 41], 1, "replicate")


@pytest.mark.parametrize("G,rope,shard", [(2, "replicate", 0), (2, "replicate", 1),
                                          (4, "replicate", 3), (4, "split", 1)])
def test_dsv3_one_shard_sampled(cuda_dev, dsv3, G, rope, shard):
    """One-shard mode (the bytes one tensor-parallel rank reads) on the whole
    DeepSeek-V3-shaped workload, in the launch configuration the benchmark
    times: every CTA pair walks several requests, so the query is reloaded
    between segments.  Sampled requests, all heads and tokens, element by
    element against the oracle's shard."""
    w = dsv3
    d = to_device(w, cuda_dev)
    out_t, lse_t = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], G, rope,
                             w.scale, shard=shard)
    torch.cuda.synchronize()
    assert tp.device_status() == 0
    out, lse = to_np(out_t), to_np(lse_t)
    assert out.shape == (w.B, w.H, 512 // G) and lse.shape == (w.B, w.H, 1)
    reqs = [0, 29, 63]
    ro, rl = O.tpla_decode_ref(as_f64(w.q)[reqs], oracle_rows(w, reqs), G, rope,
                               np.float32(w.scale), shard)
    assert_out_close(out[reqs], ro)
    assert_lse_close(lse[reqs], rl)


def test_dsv3_tpla_g2_hadamard_step_sampled(cuda_dev, dsv3):
    """The benchmark step: Hadamard-rotated q and cache, TPLA G=2 decode, V-up
    with the rotation folded into W_uv.  The oracle rotates the same bf16
    inputs itself."""
    w = dsv3
    d = to_device(w, cuda_dev)
    tp.hadamard_apply(d["q"], 512)
    tp.hadamard_apply(d["cache"], 512)
    W = w.W_uv.to(cuda_dev)
    Wt = W.transpose(1, 2).contiguous()
    tp.hadamard_apply(Wt, 512)
    Wr = Wt.transpose(1, 2).contiguous()
    out_t, lse_t = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], 2, "replicate",
                             w.scale)
    y = tp.vup_combine(out_t, Wr)
    torch.cuda.synchronize()
    assert tp.device_status() == 0
    out, lse, y = to_np(out_t), to_np(lse_t), to_np(y)
    reqs = [3, 60]
    qr = rotated_bf16(w.q[reqs])
    rows = [rotated_bf16(torch.from_numpy(r).to(torch.bfloat16)) for r in oracle_rows(w, reqs)]
    ro = check_requests(w, out, lse, reqs, 2, "replicate", q=qr, rows=rows)
    # V-up of the rotated output with the folded weights equals the oracle's
    Wf = np.swapaxes(O.hadamard_ref(np.swapaxes(as_f64(w.W_uv), 1, 2), 512), 1, 2)
    Wf = as_f64(torch.from_numpy(Wf).to(torch.bfloat16))
    assert_out_close(y[reqs], O.vup_ref(ro, Wf), what="y")


@pytest.mark.parametrize("G,rope", [(1, "replicate"), (2, "split"), (4, "replicate"),
                                    (4, "split")])
def test_kimi_sampled(cuda_dev, G, rope):
    w = make_workload("kimi")
    d = to_device(w, cuda_dev)
    out, lse = decode(d, w, G, rope)
    check_requests(w, out, lse, [2, 13], G, rope)


@pytest.mark.parametrize("G,hadamard", [(2, False), (2, True)])
def test_v2lite_whole(cuda_dev, G, hadamard):
    w = make_workload("v2lite")
    d = to_device(w, cuda_dev)
    if hadamard:
        tp.hadamard_apply(d["q"], 512)
        tp.hadamard_apply(d["cache"], 512)
    out, lse = decode(d, w, G, "replicate")
    reqs = list(range(w.B))
    if hadamard:
        qr = rotated_bf16(w.q)
        rows = [rotated_bf16(torch.from_numpy(r).to(torch.bfloat16)) for r in oracle_rows(w)]
        check_requests(w, out, lse, reqs, G, "replicate", q=qr, rows=rows)
    else:
        check_requests(w, out, lse, reqs, G, "replicate")


@pytest.fixture(scope="module")
def long_ctx():
    return make_workload("long")


@pytest.mark.parametrize("G,num_splits", [(1, 32), (1, 128), (4, 64), (1, 0)])
def test_long_context_splits_sampled(cuda_dev, long_ctx, G, num_splits):
    w = long_ctx
    d = to_device(w, cuda_dev)
    out, lse = decode(d, w, G, "replicate", num_splits=num_splits)
    check_requests(w, out, lse, [1], G, "replicate")
