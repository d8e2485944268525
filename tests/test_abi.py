"""The C-ABI library loads and exports every symbol include/tpla.h declares;
argument validation rejects bad calls before touching a GPU.  CPU only."""

import ctypes
import os
import re

import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from mla_latent_kv_dim_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "tpla.h")).read()
    return sorted(set(re.findall(r"TPLA_API\s+[\w\s\*]+?\b(tpla_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("tpla_decode", "tpla_decode_ex", "tpla_decode_workspace_size",
              "tpla_hadamard_apply", "tpla_vup_combine", "tpla_lse_merge",
              "tpla_error_string", "tpla_get_device_status", "tpla_version",
              "tpla_last_cuda_error", "tpla_launch_count"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = tp.lib()
    for n in _declared():
        assert hasattr(L, n), n
    assert tp.version() == 100


def test_error_strings():
    assert tp.error_string(0) == "ok"
    assert "invalid" in tp.error_string(-1)
    assert tp.error_string(12345) == "unknown status"


def _fake(shape, dtype, ptr=0x10000):
    """Descriptor with a fake (never dereferenced) aligned pointer."""
    d = N.TplaTensor()
    d.data = ptr
    d.dtype = {torch.bfloat16: 1, torch.float32: 2, torch.int32: 3}[dtype]
    d.ndim = len(shape)
    st = 1
    strides = []
    for s in reversed(shape):
        strides.append(st)
        st *= s
    strides = list(reversed(strides))
    for i, s in enumerate(shape):
        d.shape[i] = s
        d.stride[i] = strides[i]
    return d


def _call(q, kv, seq, pt, G, rope, out, lse, opts=None, scale=0.07):
    B = ctypes.byref
    return tp.lib().tpla_decode_ex(B(q), B(kv), B(seq), B(pt) if pt else None, G, rope,
                                   ctypes.c_float(scale), B(out), B(lse) if lse else None,
                                   B(opts) if opts else None, None)


def _good(B=2, H=16, G=2, shard=None):
    q = _fake((B, H, 576), torch.bfloat16)
    kv = _fake((8, 64, 576), torch.bfloat16)
    seq = _fake((B,), torch.int32)
    pt = _fake((B, 4), torch.int32)
    w = 512 if shard is None else 512 // G
    out = _fake((B, H, w), torch.float32)
    lse = _fake((B, H, G if shard is None else 1), torch.float32)
    return q, kv, seq, pt, out, lse


@pytest.mark.parametrize("mutate", [
    "G3", "G16", "rope2", "q_width", "q_dtype", "kv_page64", "seq_len", "out_width",
    "lse_width", "nan_scale", "q_misaligned", "q_stride", "shard_range", "reserved",
])
def test_validation_rejects_without_launch(mutate):
    q, kv, seq, pt, out, lse = _good()
    G, rope, scale, opts = 2, 0, 0.07, None
    if mutate == "G3":
        G = 3
    elif mutate == "G16":
        G = 16
    elif mutate == "rope2":
        rope = 2
    elif mutate == "q_width":
        q.shape[2] = 512
    elif mutate == "q_dtype":
        q.dtype = 2
    elif mutate == "kv_page64":
        kv.shape[1] = 32
    elif mutate == "seq_len":
        seq.shape[0] = 3
    elif mutate == "out_width":
        out.shape[2] = 256
    elif mutate == "lse_width":
        lse.shape[2] = 1
    elif mutate == "nan_scale":
        scale = float("nan")
    elif mutate == "q_misaligned":
        q.data = 0x10002
    elif mutate == "q_stride":
        q.stride[1] = 577
    elif mutate == "shard_range":
        opts = N._opts(0, 2, "auto")
    elif mutate == "reserved":
        opts = N._opts(0, None, "auto")
        opts.reserved = 1
    rc = _call(q, kv, seq, pt, G, rope, out, lse, opts, scale)
    expect = -2 if mutate == "kv_page64" else -1
    assert rc == expect, (mutate, rc)
    assert tp.launch_count() == 0


@pytest.mark.parametrize("case", ["splits", "request_heads", "request_splits",
                                  "generic_grid"])
def test_size_limits_are_unsupported_without_launch(case):
    """Sizes whose launch geometry the kernels cannot express come back as
    TPLA_ERR_UNSUPPORTED before anything is launched."""
    before = tp.launch_count()
    G, opts = 2, None
    if case == "splits":
        q, kv, seq, pt, out, lse = _good()
        opts = N._opts(65536, None, "auto")
    elif case == "request_heads":  # B * H > 2^30
        q, kv, seq, pt, out, lse = _good(B=1 << 20, H=2048)
    elif case == "request_splits":  # B * num_splits > 2^24
        q, kv, seq, pt, out, lse = _good(B=1 << 12)
        opts = N._opts(1 << 13, None, "auto")
    else:  # the portable kernel's grid: B * shards > 65535
        G = 8
        q, kv, seq, pt, out, lse = _good(B=10000, G=8)
        opts = N._opts(0, None, "generic")
    assert _call(q, kv, seq, pt, G, 0, out, lse, opts) == -2
    n = ctypes.c_size_t(0)
    rc = tp.lib().tpla_decode_workspace_size(ctypes.byref(q), ctypes.byref(kv), ctypes.byref(seq),
                                             ctypes.byref(pt), G, 0, ctypes.byref(out),
                                             ctypes.byref(opts) if opts else None,
                                             ctypes.byref(n))
    assert rc == -2
    assert tp.launch_count() == before


def test_lse_merge_size_limits():
    o = _fake((2, 1 << 16, 1 << 15, 8), torch.float32)
    lp = _fake((2, 1 << 16, 1 << 15, 1), torch.float32)
    out = _fake((1 << 16, 1 << 15, 8), torch.float32)
    assert tp.lib().tpla_lse_merge(ctypes.byref(o), ctypes.byref(lp), ctypes.byref(out), None,
                                   None) == -2
    o = _fake((1025, 1, 1, 8), torch.float32)
    lp = _fake((1025, 1, 1, 1), torch.float32)
    out = _fake((1, 1, 8), torch.float32)
    assert tp.lib().tpla_lse_merge(ctypes.byref(o), ctypes.byref(lp), ctypes.byref(out), None,
                                   None) == -2


def test_one_shard_shapes_validate():
    q, kv, seq, pt, out, lse = _good(G=4, shard=1)
    opts = N._opts(0, 1, "generic")
    n = ctypes.c_size_t(123)
    rc = tp.lib().tpla_decode_workspace_size(ctypes.byref(q), ctypes.byref(kv), ctypes.byref(seq),
                                             ctypes.byref(pt), 4, 1, ctypes.byref(out),
                                             ctypes.byref(opts), ctypes.byref(n))
    assert rc == 0
    # full-width out is rejected in one-shard mode
    q, kv, seq, pt, out, lse = _good(G=4)
    rc = tp.lib().tpla_decode_workspace_size(ctypes.byref(q), ctypes.byref(kv), ctypes.byref(seq),
                                             ctypes.byref(pt), 4, 1, ctypes.byref(out),
                                             ctypes.byref(opts), ctypes.byref(n))
    assert rc == -1


def test_generic_workspace_size_formula():
    B, H, G = 3, 16, 2
    q, kv, seq, pt, out, lse = _good(B=B, H=H, G=G)
    for splits in (1, 2, 7):
        opts = N._opts(splits, None, "generic")
        n = ctypes.c_size_t(0)
        rc = tp.lib().tpla_decode_workspace_size(ctypes.byref(q), ctypes.byref(kv),
                                                 ctypes.byref(seq), ctypes.byref(pt), G, 0,
                                                 ctypes.byref(out), ctypes.byref(opts),
                                                 ctypes.byref(n))
        assert rc == 0
        if splits == 1:
            assert n.value == 0
        else:
            o = splits * B * H * 512 * 4
            assert n.value == (o + 255) // 256 * 256 + splits * B * H * G * 4


def test_hadamard_and_vup_validation():
    L = tp.lib()
    buf = _fake((4, 576), torch.bfloat16)
    assert L.tpla_hadamard_apply(ctypes.byref(buf), 100, None) == -2
    assert L.tpla_hadamard_apply(ctypes.byref(buf), 2048, None) == -2
    small = _fake((4, 256), torch.bfloat16)
    assert L.tpla_hadamard_apply(ctypes.byref(small), 512, None) == -1
    o = _fake((2, 4, 512), torch.float32)
    W = _fake((4, 512, 100), torch.bfloat16)
    y = _fake((2, 4, 100), torch.float32)
    assert L.tpla_vup_combine(ctypes.byref(o), ctypes.byref(W), ctypes.byref(y), None) == -2
    W = _fake((3, 512, 128), torch.bfloat16)
    y = _fake((2, 4, 128), torch.float32)
    assert L.tpla_vup_combine(ctypes.byref(o), ctypes.byref(W), ctypes.byref(y), None) == -1
    # K (the contracted latent columns): a multiple of 64 up to 512, shared by out and W
    for K in (0, 32, 96, 576):
        oK = _fake((2, 4, K), torch.float32)
        WK = _fake((4, K, 128), torch.bfloat16)
        assert L.tpla_vup_combine(ctypes.byref(oK), ctypes.byref(WK), ctypes.byref(y), None) == -1
    o256 = _fake((2, 4, 256), torch.float32)
    assert L.tpla_vup_combine(ctypes.byref(o256), ctypes.byref(_fake((4, 512, 128), torch.bfloat16)),
                              ctypes.byref(y), None) == -1
    assert tp.launch_count() == 0


def test_binding_rejects_host_tensors_before_the_library():
    """The binding hands raw addresses to kernels, so host tensors are refused
    in Python before any library call."""
    before = tp.launch_count()
    q = torch.zeros((1, 16, 576), dtype=torch.bfloat16)
    cache = torch.zeros((1, 64, 576), dtype=torch.bfloat16)
    seq = torch.ones((1,), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensors"):
        tp.decode(q, cache, seq, None, 1, "replicate", 0.07)
    with pytest.raises(ValueError, match="CUDA tensors"):
        tp.hadamard_apply(torch.zeros((4, 512)), 512)
    with pytest.raises(ValueError, match="CUDA tensors"):
        tp.vup_combine(torch.zeros((1, 1, 512)), torch.zeros((1, 512, 128), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA tensors"):
        tp.lse_merge(torch.zeros((2, 1, 1, 8)), torch.zeros((2, 1, 1, 1)))
    assert tp.launch_count() == before


class _OnCuda:
    """Stands in for a CUDA tensor: only what the device check reads."""
    is_cuda = True

    def __init__(self, index):
        self.device = torch.device("cuda", index)


def test_binding_device_check(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    N._on_current_device(_OnCuda(0), None, _OnCuda(0))
    with pytest.raises(ValueError, match="different devices"):
        N._on_current_device(_OnCuda(0), _OnCuda(1))
    with pytest.raises(ValueError, match="current device"):
        N._on_current_device(_OnCuda(1), _OnCuda(1))


@pytest.mark.parametrize("B,H", [(0, 16), (2, 0)])
def test_empty_batch_or_heads_is_a_no_op(B, H):
    """No requests (or no heads) is a valid call that launches nothing."""
    before = tp.launch_count()
    q, kv, seq, pt, out, lse = _good(B=B, H=H)
    assert _call(q, kv, seq, pt, 2, 0, out, lse) == 0
    assert _call(q, kv, seq, pt, 2, 0, out, lse, N._opts(0, None, "generic")) == 0
    assert tp.launch_count() == before


def test_pca_entry_points_validate_without_launch():
    L = tp.lib()
    before = tp.launch_count()
    B = ctypes.byref
    rows = _fake((4, 64, 576), torch.bfloat16)
    C = _fake((512, 512), torch.float32)
    s = _fake((512,), torch.float32)
    U = _fake((512, 512), torch.bfloat16)
    # rows narrower than the latent, wrong dtype, misaligned
    assert L.tpla_latent_covariance(B(_fake((4, 500), torch.bfloat16)), B(C), B(s), None) == -1
    assert L.tpla_latent_covariance(B(_fake((4, 576), torch.float32)), B(C), B(s), None) == -1
    bad = _fake((4, 576), torch.bfloat16, ptr=0x10002)
    assert L.tpla_latent_covariance(B(bad), B(C), B(s), None) == -1
    assert L.tpla_latent_covariance(B(rows), B(_fake((512, 256), torch.float32)), B(s), None) == -1
    assert L.tpla_covariance_finalize(B(C), B(s), 0, B(C), B(s), None) == -1
    # U must be [512, 512] bf16 row-major; scratch must hold one leading index
    assert L.tpla_rotate_apply(B(rows), B(_fake((512, 256), torch.bfloat16)), 0x20000, 1 << 20,
                               None) == -1
    Ut = _fake((512, 512), torch.bfloat16)
    Ut.stride[0], Ut.stride[1] = 1, 512
    assert L.tpla_rotate_apply(B(rows), B(Ut), 0x20000, 1 << 20, None) == -1
    assert L.tpla_rotate_apply(B(rows), B(U), None, 1 << 20, None) == -4
    assert L.tpla_rotate_apply(B(rows), B(U), 0x20000, 64 * 512 * 4 - 16, None) == -4
    assert L.tpla_rotate_apply(B(rows), B(U), 0x20008, 1 << 20, None) == -4
    assert tp.launch_count() == before


def test_cache_append_validates_without_launch():
    L = tp.lib()
    before = tp.launch_count()
    B = ctypes.byref
    new = _fake((3, 576), torch.bfloat16)
    pos = _fake((3,), torch.int32)
    pt = _fake((3, 4), torch.int32)
    cache = _fake((10, 64, 576), torch.bfloat16)

    def call(n=new, p=pos, t=pt, c=cache, groups=2, had=1, eps=1e-6):
        return L.tpla_cache_append(B(n), B(p), B(t) if t is not None else None, B(c), groups,
                                   had, ctypes.c_float(eps), None)

    assert call(n=_fake((3, 512), torch.bfloat16)) == -1          # row width
    assert call(n=_fake((3, 576), torch.int32)) == -1             # dtype
    assert call(n=_fake((3, 576), torch.bfloat16, ptr=0x10002)) == -1  # alignment
    assert call(p=_fake((2,), torch.int32)) == -1                 # one position per request
    assert call(t=_fake((2, 4), torch.int32)) == -1               # page table rows
    assert call(c=_fake((10, 32, 576), torch.bfloat16)) == -2     # 64-token pages only
    assert call(c=_fake((10, 64, 576), torch.float32)) == -1      # bf16 cache
    assert call(groups=3) == -1 and call(groups=16) == -1
    assert call(had=2) == -1
    assert call(eps=-1.0) == -1 and call(eps=float("nan")) == -1
    assert call(t=None) == -1                                     # contiguous: [B, Lmax, 576]
    assert tp.launch_count() == before


def test_prefill_validates_without_launch():
    L = tp.lib()
    before = tp.launch_count()
    B = ctypes.byref
    q = _fake((5, 16, 576), torch.bfloat16)
    new = _fake((5, 576), torch.bfloat16)
    row = _fake((2,), torch.int32)
    cache = _fake((10, 64, 576), torch.bfloat16)
    out = _fake((5, 16, 512), torch.float32)

    def call(q=q, n=new, start=0, r=row, c=cache, groups=1, had=0, eps=1e-6, scale=0.1, o=out,
             ws=None, ws_bytes=0):
        return L.tpla_prefill(B(q), B(n), start, B(r) if r is not None else None, B(c), groups,
                              had, ctypes.c_float(eps), ctypes.c_float(scale), B(o), None, ws,
                              ws_bytes, None)

    assert call(n=_fake((4, 576), torch.bfloat16)) == -1        # one row per prompt token
    assert call(n=_fake((5, 512), torch.bfloat16)) == -1        # row width
    assert call(start=-1) == -1
    assert call(start=124) == -1                                # 124 + 5 > 2 pages
    assert call(r=None) == -1 and call(r=_fake((2, 2), torch.int32)) == -1
    assert call(c=_fake((10, 32, 576), torch.bfloat16)) == -2   # 64-token pages only
    assert call(groups=3) == -1 and call(had=2) == -1 and call(eps=-1.0) == -1
    assert call(scale=float("inf")) == -1
    assert call(o=_fake((5, 16, 256), torch.float32)) == -1     # out is [T, H, 512]
    assert call(q=_fake((5, 16, 576), torch.float32)) == -1     # bf16 queries
    assert call(q=_fake((1 << 20 + 1, 1, 576), torch.bfloat16)) == -2
    n = ctypes.c_size_t(7)
    assert L.tpla_prefill_workspace_size(None, B(n)) == -1
    assert tp.launch_count() == before
