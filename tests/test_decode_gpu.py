"""GPU parity: libtpla decode (through the C ABI) against the float64 oracle
on the same seeded inputs, element by element."""

import math

import numpy as np
import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from mla_latent_kv_dim_b200.workloads import make_inputs, make_workload
from oracle import tpla_oracle as O
from parity import (as_f64, assert_lse_close, assert_out_close, oracle_decode,
                    oracle_rows, to_device, to_np)

pytestmark = pytest.mark.gpu

KERNELS = ["generic", "sm100"]


def run(dev, w, G, rope, kernel, shard=None, num_splits=0, out_dtype=torch.float32, d=None):
    d = d or to_device(w, dev)
    try:
        out, lse = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], G, rope,
                             w.scale, shard=shard, num_splits=num_splits, kernel=kernel,
                             out_dtype=out_dtype)
    except tp.TplaError as e:
        if kernel == "sm100" and e.status == -2:
            pytest.skip("shape not covered by the tcgen05 kernel")
        raise
    torch.cuda.synchronize()
    assert tp.device_status() == 0
    return to_np(out), to_np(lse)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("G", [1, 2])
def test_tiny_config(cuda_dev, kernel, G):
    w = make_workload("tiny")
    out, lse = run(cuda_dev, w, G, "replicate", kernel)
    ro, rl = oracle_decode(w, G, "replicate")
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


RAGGED = [1, 63, 64, 65, 300, 0, 129]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("H", [16, 64, 128, 256])
@pytest.mark.parametrize("G,rope", [(1, "replicate"), (2, "replicate"), (2, "split"),
                                    (4, "replicate"), (4, "split"), (8, "replicate")])
def test_ragged_paged(cuda_dev, kernel, H, G, rope):
    w = make_inputs(len(RAGGED), H, RAGGED, paged=True, decay=True, seed=7 + G, spare_blocks=3)
    out, lse = run(cuda_dev, w, G, rope, kernel)
    ro, rl = oracle_decode(w, G, rope)
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("G,rope", [(2, "replicate"), (4, "split"), (4, "replicate")])
def test_one_shard_mode(cuda_dev, kernel, G, rope):
    w = make_inputs(4, 128, [700, 64, 1, 190], paged=True, decay=True, seed=21)
    d = to_device(w, cuda_dev)
    for s in range(G):
        out, lse = run(cuda_dev, w, G, rope, kernel, shard=s, d=d)
        ro, rl = oracle_decode(w, G, rope, shard=s)
        assert out.shape == (4, 128, 512 // G)
        assert_out_close(out, ro, what=f"shard {s}")
        assert_lse_close(lse, rl, what=f"shard {s}")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("splits", [1, 2, 3, 7])
def test_explicit_splits(cuda_dev, kernel, splits):
    w = make_inputs(3, 64, [1000, 5, 333], paged=True, decay=False, seed=31)
    out, lse = run(cuda_dev, w, 2, "replicate", kernel, num_splits=splits)
    ro, rl = oracle_decode(w, 2, "replicate")
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("kernel", KERNELS)
def test_contiguous_cache_ragged(cuda_dev, kernel):
    w = make_inputs(3, 128, [100, 256, 17], paged=False, decay=True, seed=41)
    out, lse = run(cuda_dev, w, 1, "replicate", kernel)
    ro, rl = oracle_decode(w, 1, "replicate")
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("kernel", KERNELS)
def test_bf16_output(cuda_dev, kernel):
    w = make_inputs(2, 128, [513, 64], paged=True, decay=True, seed=51)
    out, lse = run(cuda_dev, w, 2, "replicate", kernel, out_dtype=torch.bfloat16)
    ro, rl = oracle_decode(w, 2, "replicate")
    # a bf16 output stores the result in bf16: compare with the oracle's
    # result rounded the same way (round-to-nearest-even)
    ro = to_np(torch.from_numpy(ro).to(torch.bfloat16))
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("kernel", KERNELS)
def test_all_empty_and_single_token(cuda_dev, kernel):
    w = make_inputs(3, 16, [0, 1, 0], paged=True, seed=61)
    out, lse = run(cuda_dev, w, 2, "replicate", kernel)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2]))
    ro, rl = oracle_decode(w, 2, "replicate")
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("kernel", KERNELS)
def test_constant_cache_returns_row(cuda_dev, kernel):
    """Closed form on the GPU: a constant cache returns its latent row."""
    w = make_inputs(2, 64, [300, 77], paged=True, seed=71)
    w.cache[:] = w.cache[0, 0]
    out, lse = run(cuda_dev, w, 4, "split", kernel)
    row = as_f64(w.cache[0, 0])[:512]
    assert_out_close(out, np.broadcast_to(row, out.shape))


def test_convenience_entry_matches_ex(cuda_dev):
    w = make_inputs(3, 64, [900, 64, 3], paged=True, decay=True, seed=81)
    d = to_device(w, cuda_dev)
    out = torch.empty((3, 64, 512), device=cuda_dev)
    lse = torch.empty((3, 64, 2), device=cuda_dev)
    tp.decode_simple(d["q"], d["cache"], d["seq_lens"], d["page_table"], 2, "replicate",
                     w.scale, out, lse)
    torch.cuda.synchronize()
    ro, rl = oracle_decode(w, 2, "replicate")
    assert_out_close(to_np(out), ro)
    assert_lse_close(to_np(lse), rl)


@pytest.mark.parametrize("kernel", KERNELS)
def test_bad_page_id_sets_status(cuda_dev, kernel):
    """An out-of-range page id is not read: the kernel records the bounds
    error and the other requests are unaffected."""
    w = make_inputs(3, 16, [200, 100, 64], paged=True, seed=91)
    d = to_device(w, cuda_dev)
    d["page_table"][1, 0] = w.cache.shape[0] + 5
    try:
        out, lse = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], 1,
                             "replicate", w.scale, kernel=kernel)
    except tp.TplaError as e:
        if kernel == "sm100" and e.status == -2:
            pytest.skip("shape not covered by the tcgen05 kernel")
        raise
    assert tp.device_status() == -6
    assert tp.device_status() == 0  # cleared by the read
    ro, rl = oracle_decode(w, 1, "replicate", requests=[0, 2])
    o = to_np(out)
    assert_out_close(o[[0, 2]], ro)


def test_device_wait_timeout_is_reported_and_context_survives(cuda_dev):
    """A bounded barrier wait that nothing completes gives up after ~1 ms,
    records TPLA_ERR_DEVICE_TIMEOUT and returns: no hang, no fault, and the
    next decode on the same context is correct."""
    assert tp.device_status() == 0
    tp.selftest_wait_timeout(1000)
    assert tp.device_status() == -5
    assert tp.device_status() == 0  # cleared by the read
    w = make_workload("tiny")
    out, lse = run(cuda_dev, w, 1, "replicate", "sm100")
    ro, rl = oracle_decode(w, 1, "replicate")
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)


def test_hadamard_end_to_end_g1_invariance(cuda_dev):
    """Rotate q and cache on the GPU, decode exact MLA, un-rotate the output:
    equals the unrotated oracle (U U^T = I), through one bf16 re-rounding of
    the rotated inputs (tolerance factor 2)."""
    w = make_inputs(3, 64, [400, 64, 1], paged=True, decay=True, seed=101)
    d = to_device(w, cuda_dev)
    tp.hadamard_apply(d["q"], 512)
    tp.hadamard_apply(d["cache"], 512)
    out, lse = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], 1, "replicate",
                         w.scale)
    tp.hadamard_apply(out, 512)
    torch.cuda.synchronize()
    ro, rl = oracle_decode(w, 1, "replicate")
    assert_out_close(to_np(out), ro, factor=2.0)
    assert_lse_close(to_np(lse), rl, factor=2.0)


def test_hadamard_tpla_g2_matches_oracle_on_rotated_inputs(cuda_dev):
    """TPLA G=2 with the Hadamard reparameterisation: the oracle rotates the
    same bf16 inputs in float64 and rounds them to bf16 itself."""
    w = make_inputs(2, 128, [512, 130], paged=True, decay=True, seed=111)
    d = to_device(w, cuda_dev)
    tp.hadamard_apply(d["q"], 512)
    tp.hadamard_apply(d["cache"], 512)
    out, lse = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], 2, "replicate",
                         w.scale)
    torch.cuda.synchronize()
    qr = torch.from_numpy(O.hadamard_ref(as_f64(w.q), 512)).to(torch.bfloat16)
    rows = [torch.from_numpy(O.hadamard_ref(r, 512)).to(torch.bfloat16)
            for r in oracle_rows(w)]
    ro, rl = O.tpla_decode_ref(as_f64(qr), [as_f64(r) for r in rows], 2, "replicate",
                               np.float32(w.scale))
    assert_out_close(to_np(out), ro)
    assert_lse_close(to_np(lse), rl)


def test_auto_never_falls_back_to_the_portable_kernel(cuda_dev):
    """G = 8 is outside the tcgen05 kernel: the automatic choice reports
    UNSUPPORTED before any launch instead of running another kernel; the
    portable kernel runs it when named."""
    w = make_inputs(2, 16, [300, 64], paged=True, decay=True, seed=131)
    d = to_device(w, cuda_dev)
    before = tp.launch_count()
    with pytest.raises(tp.TplaError) as e:
        tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], 8, "replicate", w.scale)
    assert e.value.status == -2
    assert tp.launch_count() == before
    out, lse = run(cuda_dev, w, 8, "replicate", "generic", d=d)
    ro, rl = oracle_decode(w, 8, "replicate")
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
