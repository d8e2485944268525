"""Tensor-parallel TPLA over G ranks (one process per GPU): the deployment
the pages describe.  Rank g attends over its own shard of the latent (the
columns I_g = [g 512/G, (g+1) 512/G) plus the rope columns) with its own
softmax, multiplies its output by the rows I_g of W_uv, and the all-reduce
after the V up-projection sums the G partial products into the combined
output (feature request "Bandwidth-optimal tensor-parallel sharding of MLA",
"Directions under investigation"; TPLA abstract: attention per shard, results
combined with an all-reduce).  Head-parallel exact MLA, heads split across
ranks over the whole latent, is the baseline TPLA replaces; with G = 1 the
two are the same computation ("Tests / validation": G = 1 matches head-TP
MLA exactly).

Every step of the arithmetic runs in libtpla's kernels: the one-shard decode
(tpla_decode_ex with opts->shard = g) and the V up-projection over K = 512/G
columns (tpla_vup_combine).  This module chooses each rank's slices and calls
the collective (NCCL for CUDA tensors).

Each rank here holds the full-width cache and reads only its shard's columns,
which are the bytes a rank storing its slice alone would read; a cache laid
out with 512/G + 64 columns per token is not built.
"""
from __future__ import annotations

from ._native import decode, vup_combine

LATENT = 512


def shard_columns(G: int, rank: int) -> slice:
    """Latent columns of rank `rank` out of G (contiguous blocks, shard order)."""
    if G not in (1, 2, 4, 8) or not 0 <= rank < G:
        raise ValueError("G must be 1, 2, 4 or 8 and 0 <= rank < G")
    d = LATENT // G
    return slice(rank * d, (rank + 1) * d)


def shard_weights(W_uv, G: int, rank: int):
    """Rows I_g of W_uv [H, 512, Dv]: a view, no copy."""
    return W_uv[:, shard_columns(G, rank), :]


def rank_partial(q, kv_cache, seq_lens, page_table, G, rank, W_uv, scale,
                 rope_mode="replicate", workspace=None, stream=None):
    """Rank `rank`'s share of one TPLA decode step.

    Returns (y_g, out_g, lse_g): the partial product y_g = out_g W_uv[:, I_g, :]
    ([B, H, Dv] f32), the rank's attention output over its shard
    ([B, H, 512/G] f32) and its lse ([B, H, 1])."""
    out, lse = decode(q, kv_cache, seq_lens, page_table, G, rope_mode, scale,
                      shard=rank if G > 1 else None, workspace=workspace, stream=stream)
    y = vup_combine(out, shard_weights(W_uv, G, rank), stream=stream)
    return y, out, lse


def all_reduce_partials(y, group=None):
    """Sum the ranks' partial products in place over the process group (the
    all-reduce after the V up-projection); unchanged without a group."""
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


def tpla_step(q, kv_cache, seq_lens, page_table, W_uv, scale, group=None,
              rope_mode="replicate", workspace=None, stream=None):
    """One TPLA decode step on this rank: G = the group's size, shard = the
    rank; returns the combined y [B, H, Dv] (every rank holds it)."""
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        G, rank = dist.get_world_size(group), dist.get_rank(group)
    else:
        G, rank = 1, 0
    y, _, _ = rank_partial(q, kv_cache, seq_lens, page_table, G, rank, W_uv, scale,
                           rope_mode, workspace, stream)
    return all_reduce_partials(y, group)


def head_slice(H: int, world: int, rank: int) -> slice:
    """Heads of rank `rank` when H heads are split evenly over `world` ranks."""
    if world < 1 or H % world or not 0 <= rank < world:
        raise ValueError("the heads must split evenly over the ranks")
    h = H // world
    return slice(rank * h, (rank + 1) * h)


def head_parallel_partial(q, kv_cache, seq_lens, page_table, W_uv, scale, world, rank,
                          workspace=None, stream=None):
    """Exact MLA with heads split across ranks: rank `rank` decodes its heads
    over the whole latent and projects them.  Returns (y_r [B, H/world, Dv],
    out_r [B, H/world, 512], lse_r); the full y is the concatenation over
    ranks along the heads (an all-gather)."""
    hs = head_slice(q.shape[1], world, rank)
    out, lse = decode(q[:, hs], kv_cache, seq_lens, page_table, 1, "replicate", scale,
                      workspace=workspace, stream=stream)
    y = vup_combine(out, W_uv[hs], stream=stream)
    return y, out, lse
