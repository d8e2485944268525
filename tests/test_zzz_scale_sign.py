"""Decode with a scale <= 0 under the automatic kernel choice: the tcgen05
kernel takes positive scales only, so the call runs the generic kernel, and
the workspace the size query returns has to cover that kernel too.  The case
is chosen so that the generic kernel's split count (64 chunks of a 16K-token
request) needs more scratch than the tcgen05 kernel's slots.  Collected
after the other GPU tests."""

import numpy as np
import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from mla_latent_kv_dim_b200.workloads import make_inputs
from oracle import tpla_oracle as O
from parity import (as_f64, assert_lse_close, assert_out_close, oracle_rows, to_device,
                    to_np)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sign", [-1.0, 0.0])
def test_nonpositive_scale_runs_generic_with_enough_workspace(cuda_dev, sign):
    w = make_inputs(4, 16, [16384, 5, 9000, 0], paged=True, decay=True, seed=21)
    d = to_device(w, cuda_dev)
    scale = float(np.float32(sign * w.scale))
    out = torch.empty((w.B, w.H, 512), device=cuda_dev)
    need_auto = tp.decode_workspace_size(d["q"], d["cache"], d["seq_lens"], d["page_table"], 1,
                                         "replicate", out)
    need_generic = tp.decode_workspace_size(d["q"], d["cache"], d["seq_lens"], d["page_table"],
                                            1, "replicate", out, kernel="generic")
    assert need_auto >= need_generic > 0
    out, lse = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], 1, "replicate",
                         scale)
    torch.cuda.synchronize()
    assert tp.device_status() == 0
    ro, rl = O.tpla_decode_ref(as_f64(w.q), oracle_rows(w), 1, "replicate", np.float32(scale))
    assert_out_close(to_np(out), ro)
    assert_lse_close(to_np(lse), rl)
