"""Decode with a scale <= 0 under the automatic kernel choice: the tcgen05
kernel takes any finite scale (a negative one negates the scores before the
row max; zero gives uniform weights), so no other kernel runs, and the size
query for the automatic choice equals the tcgen05 kernel's.  Collected after
the other GPU tests."""

import numpy as np
import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from mla_latent_kv_dim_b200.workloads import make_inputs
from oracle import tpla_oracle as O
from parity import (as_f64, assert_lse_close, assert_out_close, oracle_rows, to_device,
                    to_np)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sign,G", [(-1.0, 1), (0.0, 1), (-1.0, 2), (0.0, 4)])
def test_nonpositive_scale_runs_tcgen05(cuda_dev, sign, G):
    w = make_inputs(4, 16, [16384, 5, 9000, 0], paged=True, decay=True, seed=21)
    d = to_device(w, cuda_dev)
    scale = float(np.float32(sign * w.scale))
    out = torch.empty((w.B, w.H, 512), device=cuda_dev)
    need_auto = tp.decode_workspace_size(d["q"], d["cache"], d["seq_lens"], d["page_table"], G,
                                         "replicate", out)
    need_sm100 = tp.decode_workspace_size(d["q"], d["cache"], d["seq_lens"], d["page_table"],
                                          G, "replicate", out, kernel="sm100")
    assert need_auto == need_sm100 > 0
    before = tp.launch_count()
    out, lse = tp.decode(d["q"], d["cache"], d["seq_lens"], d["page_table"], G, "replicate",
                         scale)
    torch.cuda.synchronize()
    assert tp.launch_count() - before == 2  # the tcgen05 kernel and its merge
    assert tp.device_status() == 0
    ro, rl = O.tpla_decode_ref(as_f64(w.q), oracle_rows(w), G, "replicate", np.float32(scale))
    assert_out_close(to_np(out), ro)
    assert_lse_close(to_np(lse), rl)
