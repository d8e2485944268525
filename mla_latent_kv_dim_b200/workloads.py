"""Seeded synthetic decode workloads (inputs only).

This module draws random inputs and lays them out; it holds none of the
method's arithmetic.  The same arrays feed the CUDA path and the CPU oracle.

Recipe (fixed order, one NumPy PCG64 stream per workload seed):

1. ``seq_lens``: a fixed length, or integers uniform in [lo, hi] inclusive;
2. ``q`` [B, H, 576] ~ N(0, 1);
3. cache rows [num_blocks, 64, 576] (paged) or [B, Lmax, 576] (contiguous)
   ~ N(0, 1), latent channel j (0..511) multiplied by exp(-j / 128) when
   ``decay`` is on (rope channels are not scaled);
4. paged caches only: ``perm = rng.permutation(num_blocks)``; logical page p
   of request b is physical block ``perm[first_page[b] + p]``;
5. ``W_uv`` [H, 512, 128] ~ N(0, 0.02) when requested.

Prefill inputs (``make_prefill_inputs``), one request: ``q`` [T, H, 576]
~ N(0, 1); the prompt's new rows ``kv_new`` [T, 576] drawn like cache rows
(float32, not rounded); a paged cache whose rows (the ``start`` tokens cached
before the prompt, and unused rows) are drawn like cache rows; the request's
page row is the first pages of ``rng.permutation(num_blocks)``.

Values are drawn in float32 and rounded to bf16 (round-to-nearest-even).
The named workloads are DeepSeek-V2-Lite, DeepSeek-V3 and Kimi-K2-shaped
stand-ins (no checkpoints or datasets are used).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

LATENT = 512
ROPE = 64
WIDTH = 576
BLOCK = 64
V_HEAD = 128
SOFTMAX_SCALE = 1.0 / math.sqrt(192.0)  # DeepSeek qk_nope 128 + qk_rope 64

_GEN_CHUNK_ROWS = 1 << 16  # rows drawn per NumPy call for large caches


@dataclass
class Workload:
    name: str
    B: int
    H: int
    seq_lens: torch.Tensor          # [B] int32
    q: torch.Tensor                 # [B, H, 576] bf16
    cache: torch.Tensor             # [num_blocks, 64, 576] or [B, Lmax, 576] bf16
    page_table: torch.Tensor | None  # [B, max_pages] int32 (paged only)
    W_uv: torch.Tensor | None       # [H, 512, 128] bf16
    scale: float = SOFTMAX_SCALE
    meta: dict = field(default_factory=dict)

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    def latent_kv_bytes(self, G: int = 1, shard: int | None = None,
                        rope_mode: str = "replicate") -> int:
        """Algorithmic cache bytes one decode step must read: every cached
        value of the columns it needs, once (rope shared across shards)."""
        if shard is None:
            per_tok = WIDTH * 2
        else:
            rope = ROPE if rope_mode == "replicate" else ROPE // G
            per_tok = (LATENT // G + rope) * 2
        return int(self.seq_lens.to(torch.int64).sum().item()) * per_tok


# Named workloads.  lens: ("fixed", L) or ("uniform", lo, hi).
CONFIGS = {
    "tiny": dict(B=1, H=16, lens=("fixed", 256), paged=False, decay=False,
                 seed=0, wuv=False),
    "v2lite": dict(B=32, H=16, lens=("uniform", 2048, 4096), paged=True,
                   decay=True, seed=1, wuv=True),
    "dsv3": dict(B=64, H=128, lens=("fixed", 32768), paged=True, decay=True,
                 seed=2, wuv=True),
    "kimi": dict(B=16, H=64, lens=("uniform", 16384, 32768), paged=True,
                 decay=True, seed=3, wuv=True),
    "long": dict(B=4, H=128, lens=("fixed", 131072), paged=True, decay=True,
                 seed=4, wuv=False),
}


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _draw_rows(rng, n_rows: int, decay: bool, out: torch.Tensor) -> None:
    """Fill ``out`` (viewed as [n_rows, 576] bf16) with N(0,1) rows."""
    flat = out.view(n_rows, WIDTH)
    scale = np.exp(-np.arange(LATENT, dtype=np.float64) / 128.0).astype(np.float32)
    for r0 in range(0, n_rows, _GEN_CHUNK_ROWS):
        r1 = min(n_rows, r0 + _GEN_CHUNK_ROWS)
        x = rng.standard_normal((r1 - r0, WIDTH), dtype=np.float32)
        if decay:
            x[:, :LATENT] *= scale
        flat[r0:r1] = _to_bf16(x)


def make_inputs(B: int, H: int, lens, *, paged: bool = True, decay: bool = False,
                seed: int = 0, wuv: bool = False, name: str = "custom",
                pin: bool = False, spare_blocks: int = 0) -> Workload:
    """Build one seeded workload.  ``lens`` is ("fixed", L), ("uniform", lo,
    hi) or an explicit list of B lengths.  ``spare_blocks`` adds unused
    physical blocks (paged caches only)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if isinstance(lens, tuple) and lens[0] == "fixed":
        seq = np.full((B,), int(lens[1]), dtype=np.int64)
    elif isinstance(lens, tuple) and lens[0] == "uniform":
        seq = rng.integers(int(lens[1]), int(lens[2]), size=B, endpoint=True)
    else:
        seq = np.asarray(list(lens), dtype=np.int64)
        assert seq.shape == (B,)
    q = _to_bf16(rng.standard_normal((B, H, WIDTH), dtype=np.float32))

    pages = [(int(L) + BLOCK - 1) // BLOCK for L in seq]
    if paged:
        num_blocks = sum(pages) + spare_blocks
        cache = torch.empty((max(num_blocks, 1), BLOCK, WIDTH), dtype=torch.bfloat16,
                            pin_memory=pin)
        _draw_rows(rng, max(num_blocks, 1) * BLOCK, decay, cache)
        perm = rng.permutation(max(num_blocks, 1))
        max_pages = max(1, max(pages) if pages else 1)
        pt = np.zeros((B, max_pages), dtype=np.int32)
        off = 0
        for b, n in enumerate(pages):
            pt[b, :n] = perm[off:off + n]
            off += n
        page_table = torch.from_numpy(pt)
    else:
        Lmax = max(1, int(seq.max()) if B else 1)
        cache = torch.empty((B, Lmax, WIDTH), dtype=torch.bfloat16, pin_memory=pin)
        _draw_rows(rng, B * Lmax, decay, cache)
        page_table = None
    W = None
    if wuv:
        W = _to_bf16(0.02 * rng.standard_normal((H, LATENT, V_HEAD), dtype=np.float32))
    return Workload(name=name, B=B, H=H,
                    seq_lens=torch.from_numpy(seq.astype(np.int32)),
                    q=q, cache=cache, page_table=page_table, W_uv=W,
                    meta=dict(seed=seed, decay=decay, paged=paged))


@dataclass
class PrefillInputs:
    start: int
    q: torch.Tensor         # [T, H, 576] bf16
    kv_new: torch.Tensor    # [T, 576] f32
    cache: torch.Tensor     # [num_blocks, 64, 576] bf16
    page_row: torch.Tensor  # [pages] int32
    scale: float = SOFTMAX_SCALE


def make_prefill_inputs(T: int, H: int, start: int = 0, *, seed: int = 0,
                        spare_blocks: int = 1, decay: bool = True) -> PrefillInputs:
    """One request's prompt of T tokens after ``start`` cached tokens."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _to_bf16(rng.standard_normal((T, H, WIDTH), dtype=np.float32))
    new = rng.standard_normal((T, WIDTH), dtype=np.float32)
    if decay:
        new[:, :LATENT] *= np.exp(-np.arange(LATENT, dtype=np.float64) / 128.0).astype(np.float32)
    pages = max(1, (start + T + BLOCK - 1) // BLOCK)
    nblk = pages + spare_blocks
    cache = torch.empty((nblk, BLOCK, WIDTH), dtype=torch.bfloat16)
    _draw_rows(rng, nblk * BLOCK, decay, cache)
    row = rng.permutation(nblk)[:pages].astype(np.int32)
    return PrefillInputs(start=start, q=q, kv_new=torch.from_numpy(new), cache=cache,
                         page_row=torch.from_numpy(row))


def make_workload(name: str, pin: bool = False, batch: int | None = None) -> Workload:
    """A named workload; ``batch`` keeps the per-request recipe with fewer
    requests (small profiling captures)."""
    c = CONFIGS[name]
    B = c["B"] if batch is None else int(batch)
    return make_inputs(B, c["H"], c["lens"], paged=c["paged"],
                       decay=c["decay"], seed=c["seed"], wuv=c["wuv"],
                       name=name, pin=pin)


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16/fp32 tensor (for the oracle side)."""
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)
