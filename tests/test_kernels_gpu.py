"""GPU parity of the auxiliary kernels (LSE merge, Hadamard, V-up combine)
against the float64 oracle."""

import math

import numpy as np
import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from oracle import tpla_oracle as O
from parity import assert_lse_close, assert_out_close, to_np

pytestmark = pytest.mark.gpu


def _bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (scale * torch.randn(shape, generator=g)).to(torch.bfloat16)


@pytest.mark.parametrize("S,Gs", [(1, 1), (3, 2), (17, 4), (128, 1)])
def test_lse_merge(cuda_dev, S, Gs):
    B, H, Wd = 3, 5, 512
    g = torch.Generator().manual_seed(S * 10 + Gs)
    o = torch.randn((S, B, H, Wd), generator=g)
    l = 3 * torch.randn((S, B, H, Gs), generator=g)
    # empty chunks (-inf) and one request with every chunk empty
    l[0, 0] = -math.inf
    l[:, 2, 1] = -math.inf
    out, lse = tp.lse_merge(o.to(cuda_dev), l.to(cuda_dev))
    torch.cuda.synchronize()
    on = o.numpy().astype(np.float64).reshape(S, B, H, Gs, Wd // Gs)
    ro, rl = O.lse_merge_ref(on, l.numpy().astype(np.float64))
    ro = ro.reshape(B, H, Wd)
    assert_out_close(to_np(out), ro)
    assert_lse_close(to_np(lse), rl)
    assert np.all(to_np(out)[2, 1] == 0)


@pytest.mark.parametrize("dim", [32, 64, 128, 256, 512, 1024])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_hadamard_matches_matrix(cuda_dev, dim, dtype):
    x = _bf16((37, dim + 64), dim).to(dtype)
    ref = O.hadamard_ref(x.double().numpy(), dim)
    y = x.to(cuda_dev)
    tp.hadamard_apply(y, dim)
    torch.cuda.synchronize()
    got = to_np(y)
    # bf16 rows are rounded once on store: compare within 2^-8 relative
    tol = 1e-5 if dtype == torch.float32 else 2 ** -8
    assert np.all(got[:, dim:] == x[:, dim:].double().numpy())
    assert np.abs(got - ref).max() <= tol * np.abs(ref).max()


def test_hadamard_strided_3d_and_involution(cuda_dev):
    base = _bf16((4, 9, 600), 5).float()
    view = base.to(cuda_dev)[:, 1:8, :576]  # strided rows
    orig = view.clone()
    tp.hadamard_apply(view, 512)
    ref = O.hadamard_ref(orig.cpu().double().numpy(), 512)
    assert np.abs(to_np(view) - ref).max() < 1e-5
    tp.hadamard_apply(view, 512)
    torch.cuda.synchronize()
    assert torch.allclose(view, orig, atol=1e-5)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,Dv", [(1, 16, 128), (64, 128, 128), (17, 64, 64), (70, 3, 256)])
def test_vup_combine(cuda_dev, out_dtype, B, H, Dv):
    g = torch.Generator().manual_seed(B * H + Dv)
    out = (torch.randn((B, H, 512), generator=g) * 0.3).to(out_dtype)
    W = (0.02 * torch.randn((H, 512, Dv), generator=g)).to(torch.bfloat16)
    y = tp.vup_combine(out.to(cuda_dev), W.to(cuda_dev))
    torch.cuda.synchronize()
    ref = O.vup_ref(out.double().numpy(), W.double().numpy())
    assert_out_close(to_np(y), ref, what="y")
    # and equal to the sum of per-shard partial products (all-reduce form)
    ref2 = O.vup_sharded_ref(out.double().numpy(), W.double().numpy(), 4)
    assert_out_close(to_np(y), ref2, what="y (sharded)")
