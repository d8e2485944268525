"""tpla_decode_noalloc: the decode entry point for callers that cannot
allocate device memory while they decode (its split-KV scratch is a fixed
buffer the library reserves when it is loaded).  Checked through the C ABI
against tpla_decode_ex, which takes caller-allocated workspace, and against
the float64 oracle, on two calls in a row that both need scratch; a call
after the first must not change the device's free memory.  Kept in a file of
its own, collected last."""

import ctypes

import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from mla_latent_kv_dim_b200 import _native as N
from mla_latent_kv_dim_b200.workloads import make_inputs
from parity import (assert_lse_close, assert_out_close, oracle_decode, to_device,
                    to_np)

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 64 * 1024 * 1024


def _noalloc(d, G, rope, scale, out, lse, num_splits, shard=None):
    L = tp.lib()
    L.tpla_decode_noalloc.argtypes = [ctypes.POINTER(N.TplaTensor)] * 4 + [
        ctypes.c_int, ctypes.c_int, ctypes.c_float] + [ctypes.POINTER(N.TplaTensor)] * 2 + [
        ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    L.tpla_decode_noalloc.restype = ctypes.c_int
    ref = lambda t: ctypes.byref(N.desc(t)) if t is not None else None  # noqa: E731
    return L.tpla_decode_noalloc(ref(d["q"]), ref(d["cache"]), ref(d["seq_lens"]),
                                 ref(d["page_table"]), G, N.ROPE_MODES[rope],
                                 ctypes.c_float(scale), ref(out), ref(lse), num_splits,
                                 -1 if shard is None else shard,
                                 torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("case", [
    dict(B=3, H=64, lens=[900, 64, 333], G=2, rope="replicate", splits=3, shard=None, seed=3),
    dict(B=4, H=128, lens=[1500, 1, 700, 64], G=4, rope="split", splits=0, shard=None, seed=4),
    dict(B=2, H=16, lens=[2000, 129], G=2, rope="replicate", splits=5, shard=1, seed=5),
])
def test_noalloc_matches_decode_ex_twice(cuda_dev, case):
    w = make_inputs(case["B"], case["H"], case["lens"], paged=True, decay=True, seed=case["seed"])
    G, rope, shard = case["G"], case["rope"], case["shard"]
    width = 512 if shard is None else 512 // G
    nsh = G if shard is None else 1
    d = to_device(w, cuda_dev)
    need = tp.decode_workspace_size(d["q"], d["cache"], d["seq_lens"], d["page_table"], G,
                                    rope, torch.empty((w.B, w.H, width), device=cuda_dev),
                                    num_splits=case["splits"], shard=shard)
    assert 0 < need <= SCRATCH_LIMIT  # the case really uses scratch
    ref_out, ref_lse = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], G, rope,
                                 w.scale, num_splits=case["splits"], shard=shard)
    ora_out, ora_lse = oracle_decode(w, G, rope, shard=shard)
    for call in range(2):
        out = torch.full((w.B, w.H, width), float("nan"), device=cuda_dev)
        lse = torch.full((w.B, w.H, nsh), float("nan"), device=cuda_dev)
        rc = _noalloc(d, G, rope, w.scale, out, lse, case["splits"], shard)
        assert rc == 0, tp.error_string(rc)
        torch.cuda.synchronize()
        assert_out_close(to_np(out), to_np(ref_out), what=f"call {call}")
        assert_lse_close(to_np(lse), to_np(ref_lse), what=f"call {call}")
        assert_out_close(to_np(out), ora_out, what=f"call {call} vs oracle")
        assert_lse_close(to_np(lse), ora_lse, what=f"call {call} vs oracle")


def test_noalloc_reserves_nothing_after_its_first_call(cuda_dev):
    """The first call on a device is the set-up call (it may load the fixed
    buffer); a later call must leave the device's free memory unchanged."""
    w = make_inputs(3, 64, [900, 64, 333], paged=True, decay=True, seed=7)
    d = to_device(w, cuda_dev)
    out = torch.empty((w.B, w.H, 512), device=cuda_dev)
    lse = torch.empty((w.B, w.H, 2), device=cuda_dev)
    assert _noalloc(d, 2, "replicate", w.scale, out, lse, 3) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert _noalloc(d, 2, "replicate", w.scale, out, lse, 3) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_dev):
    w = make_inputs(8, 128, [4096] * 8, paged=True, seed=9)
    d = to_device(w, cuda_dev)
    out = torch.empty((8, 128, 512), device=cuda_dev)
    lse = torch.empty((8, 128, 1), device=cuda_dev)
    # 64 explicit splits need 64 * 8 * 128 * 512 * 4 bytes of partials (> 64 MiB)
    before = tp.launch_count()
    rc = _noalloc(d, 1, "replicate", w.scale, out, lse, 64)
    assert rc == -4  # TPLA_ERR_WORKSPACE
    assert tp.launch_count() == before
