"""GPU parity of the tensor-parallel TPLA rank step, with the G ranks run one
after another on one GPU: each rank's one-shard decode and its partial V
up-projection (K = 512/G) against the float64 oracle, their sum (what the
all-reduce forms) against the oracle's combined output, and head-parallel
exact MLA against the whole decode (G = 1 equals head-TP MLA)."""
import numpy as np
import pytest
import torch

import mla_latent_kv_dim_b200 as tp
from mla_latent_kv_dim_b200 import tensor_parallel as T
from mla_latent_kv_dim_b200.workloads import as_f64, make_inputs
from oracle import tpla_oracle as O
from parity import assert_out_close, oracle_rows, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,H", [(2, 128), (4, 64), (2, 16)])
def test_rank_partials_sum_to_the_combined_output(cuda_dev, G, H):
    w = make_inputs(3, H, [700, 65, 300], paged=True, decay=True, seed=40 + G, wuv=True)
    q, cache = w.q.to(cuda_dev), w.cache.to(cuda_dev)
    seq, pt, W = w.seq_lens.to(cuda_dev), w.page_table.to(cuda_dev), w.W_uv.to(cuda_dev)
    rows = oracle_rows(w)
    full, _ = O.tpla_decode_ref(as_f64(w.q), rows, G, "replicate", np.float32(w.scale))
    Wf = as_f64(w.W_uv)
    total = None
    for g in range(G):
        y, out, lse = T.rank_partial(q, cache, seq, pt, G, g, W, w.scale)
        torch.cuda.synchronize()
        cols = T.shard_columns(G, g)
        og, _ = O.tpla_decode_ref(as_f64(w.q), rows, G, "replicate", np.float32(w.scale), shard=g)
        assert_out_close(to_np(out), og, what=f"rank {g} out")
        assert_out_close(to_np(y), O.vup_ref(og, Wf[:, cols, :]), what=f"rank {g} y")
        total = y.clone() if total is None else total + y
    assert tp.device_status() == 0
    assert_out_close(to_np(total), O.vup_ref(full, Wf), what="sum over ranks")


def test_head_parallel_mla_is_the_whole_decode(cuda_dev):
    """G = 1: the two heads halves of a head-parallel step give exactly the
    heads of the whole decode (every head is computed alone)."""
    w = make_inputs(2, 128, [513, 90], paged=True, decay=True, seed=44, wuv=True)
    q, cache = w.q.to(cuda_dev), w.cache.to(cuda_dev)
    seq, pt, W = w.seq_lens.to(cuda_dev), w.page_table.to(cuda_dev), w.W_uv.to(cuda_dev)
    out, lse = tp.decode(q, cache, seq, pt, 1, "replicate", w.scale)
    y = tp.vup_combine(out, W)
    yT, _, _ = T.rank_partial(q, cache, seq, pt, 1, 0, W, w.scale)  # TPLA with G = 1
    for r in range(2):
        yr, outr, lser = T.head_parallel_partial(q, cache, seq, pt, W, w.scale, 2, r)
        hs = T.head_slice(128, 2, r)
        torch.cuda.synchronize()
        assert torch.equal(outr, out[:, hs]) and torch.equal(lser, lse[:, hs])
        assert torch.equal(yr, y[:, hs])
    assert torch.equal(yT, y)
    ro, _ = O.mla_decode_ref(as_f64(w.q), oracle_rows(w), np.float32(w.scale))
    assert_out_close(to_np(y), O.vup_ref(ro, as_f64(w.W_uv)))
