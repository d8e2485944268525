"""CPU float64 oracle for MLA latent-KV decode attention and its TPLA variant.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the tests, the ``smoke()`` entry point and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code with the CUDA path
(no kernels, headers, helpers or constants); both sides only see the same
seeded input arrays.

Everything here is the plain definition, written out in float64 NumPy with no
blocking, fusion or reordering beyond what the definitions state.  Inputs are
the bf16 values of the GPU inputs widened exactly to float64; ``scale`` is the
float32 value the caller passes, widened.

Sources (web pages on TPLA / MLA latent-cache sharding):

* [ISSUE]  "[Feature Request] Bandwidth-optimal tensor-parallel sharding of MLA
  (latent-cache sharding / TPLA)", sections "Background / problem",
  "Directions under investigation", "Methodology (first step)",
  "Tests / validation".
* [ABSTRACT] "TPLA: Tensor Parallel Latent Attention for Efficient
  Disaggregated Prefill & Decode Inference", abstract.
* [REVIEW] pith.science review of arXiv 2508.15881: skeptic critique
  (load-bearing attack on Eq. 6), referee report (significance; major comments
  on Eq. 22/25), pith extraction (key machinery), desk-editor letter.

Readings taken where the pages are silent:

1. Eq. 6 is not printed; the reviewers state it is an *unscaled* local
   softmax.  Shard g therefore uses the same ``scale`` as exact MLA and no
   mu/nu factors.
2. Shard g owns the contiguous latent columns [g*d, (g+1)*d), d = 512/G.
3. Rope columns are replicated to every shard ("320 = 256 + 64 at TP=2");
   the ``split`` rope mode gives shard g the contiguous rope slice
   [512 + g*64/G, 512 + (g+1)*64/G).
4. Values are latent columns only (the rope part is key-only in MLA); the
   output lives in latent space.
5. Shard outputs are concatenated in shard order; the all-reduce becomes a
   sum over shards inside the V up-projection.
6. lse is the natural log of sum(exp(scale * logits)); an empty request has
   output 0 and lse = -inf.
7. The Hadamard transform is the orthonormal Sylvester (natural-order) matrix
   applied to the first ``dim`` columns of a row.
8. PCA is taken over the calibration rows' latent columns only (position
   features excluded): the covariance of the mean-centred rows,
   (1/N) sum (f - m)^T (f - m).  U holds the unit eigenvectors as columns in
   descending eigenvalue order, each signed so that its entry of largest
   magnitude (the first such, on a tie) is positive.  Only the rotation
   x -> x U is applied to q and the cache; the mean is not subtracted.
9. Eq. (25)'s alpha and beta are the shares of the eigenvalue sum in shard
   0's and shard 1's index ranges, taken disjoint ([0, d) and [d, 2d)), which
   fixes the overlap at lambda_{d/2} the referee points out; for G shards
   each shard's share is taken the same way.  They are diagnostics: the
   deployed computation is the unscaled local softmax (reading 1), so no
   mu/nu factor enters it.
10. The cache stores the latent after its RMS normalisation; the norm's
   learned gain is absorbed into the up-projections (like the rotation U,
   [REVIEW pith_extraction.key_machinery]), so a stored row is x / rms(x),
   taken over each of ``norm_groups`` contiguous shards (one group: exact
   MLA; G groups: every TPLA rank normalises its own slice).  The rotation,
   when used, comes first; eps is added to the mean square.
11. Prefill/decode separation ([ABSTRACT]: MLA-style prefilling, then
   tensor-parallel decoding; [REVIEW referee_report.major_comments] on Table
   2: the separated variant runs unmodified MLA during prefill and TPLA only
   during decode).  The prefill of a request stores its prompt rows through
   the cache-write step of reading 10 and gives every prompt token the exact
   MLA attention (one softmax over all 576 values per token) over the
   request's stored rows up to and including its own position (causal).  It
   is written in the absorbed form the decode uses; the per-head
   up-projected form of MLA is the same function in exact arithmetic.
"""

from __future__ import annotations

import math

import numpy as np

LATENT = 512  # kv_lora_rank: the latent part of a cache row
ROPE = 64     # decoupled rope key part of a cache row
WIDTH = LATENT + ROPE  # 576 values per token ([ISSUE] "Background / problem")
BLOCK = 64    # tokens per cache page


# ---------------------------------------------------------------------------
# Column bookkeeping for the TPLA shards
# ---------------------------------------------------------------------------

def shard_columns(G: int, g: int, rope_mode: str = "replicate"):
    """Return (latent_cols, rope_cols) of shard ``g`` out of ``G``.

    [ABSTRACT]: the latent vector, and with it the matching slice of every
    head's query, is cut into per-device pieces.  [REVIEW
    referee_report.significance]:
    the per-device cache is 256 + 64 = 320 dims at TP=2, so the rope part is
    replicated to every shard.  ``split`` (rope also cut into G slices) is
    the alternative reading; contiguous slices in shard order (readings 2, 3).
    """
    if LATENT % G:
        raise ValueError("G must divide 512")
    d = LATENT // G
    lat = np.arange(g * d, (g + 1) * d)
    if rope_mode == "replicate":
        rope = np.arange(LATENT, WIDTH)
    elif rope_mode == "split":
        if ROPE % G:
            raise ValueError("split rope needs G | 64")
        r = ROPE // G
        rope = np.arange(LATENT + g * r, LATENT + (g + 1) * r)
    else:
        raise ValueError(rope_mode)
    return lat, rope


# ---------------------------------------------------------------------------
# Cache addressing (pure indexing, no arithmetic of the method)
# ---------------------------------------------------------------------------

def gather_request_rows(cache, seq_lens, page_table=None):
    """Return a list with the [L_b, 576] float64 cache rows of each request.

    Paged: token t of request b lives in block ``page_table[b][t // 64]`` at
    row ``t % 64`` of a [num_blocks, 64, 576] cache.  Contiguous: a
    [B, Lmax, 576] cache, request b's first L_b rows.
    """
    cache = np.asarray(cache)
    rows = []
    for b, L in enumerate(np.asarray(seq_lens).tolist()):
        if page_table is None:
            rows.append(np.asarray(cache[b, :L], dtype=np.float64))
        else:
            t = np.arange(L)
            blk = np.asarray(page_table)[b][t // BLOCK]
            rows.append(np.asarray(cache[blk, t % BLOCK], dtype=np.float64))
    return rows


# ---------------------------------------------------------------------------
# The attention primitive: softmax attention of a few query rows
# ---------------------------------------------------------------------------

def attention_ref(qh, keys, values, scale):
    """Softmax attention for one request and one key/value column set.

    qh [H, K], keys [L, K], values [L, V].  s = scale * qh keys^T,
    out = softmax(s) values, lse = log sum exp(s) (natural log).
    An empty key set gives out = 0, lse = -inf (reading 6).
    """
    qh = np.asarray(qh, dtype=np.float64)
    H = qh.shape[0]
    V = values.shape[1]
    if keys.shape[0] == 0:
        return np.zeros((H, V)), np.full((H,), -np.inf)
    s = float(scale) * (qh @ np.asarray(keys, dtype=np.float64).T)  # [H, L]
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    z = p.sum(axis=1, keepdims=True)
    out = (p @ np.asarray(values, dtype=np.float64)) / z
    lse = (m + np.log(z))[:, 0]
    return out, lse


def attention_bruteforce(qh, keys, values, scale):
    """Scalar-loop restatement of ``attention_ref`` for tiny inputs.

    Pure Python floats and ``math.exp``; used only to pin the NumPy version.
    """
    H = len(qh)
    L = len(keys)
    V = len(values[0]) if L else 0
    out = [[0.0] * V for _ in range(H)]
    lse = [-math.inf] * H
    for h in range(H):
        if L == 0:
            continue
        s = []
        for t in range(L):
            acc = 0.0
            for j in range(len(qh[h])):
                acc += float(qh[h][j]) * float(keys[t][j])
            s.append(float(scale) * acc)
        m = max(s)
        w = [math.exp(x - m) for x in s]
        z = sum(w)
        for v in range(V):
            out[h][v] = sum(w[t] * float(values[t][v]) for t in range(L)) / z
        lse[h] = m + math.log(z)
    return out, lse


# ---------------------------------------------------------------------------
# Exact MLA decode (absorbed form) and TPLA
# ---------------------------------------------------------------------------

def mla_decode_ref(q, rows, scale):
    """Exact absorbed MLA decode: one new token per request.

    Every head attends over all 576 cached values per token (512 latent +
    64 rope; [ISSUE] "Background / problem") with one softmax; values are
    the 512 latent columns, so the output stays in latent space.
    q [B, H, 576]; rows: per-request [L_b, 576].  Returns out [B, H, 512],
    lse [B, H].
    """
    q = np.asarray(q, dtype=np.float64)
    B, H, _ = q.shape
    out = np.zeros((B, H, LATENT))
    lse = np.zeros((B, H))
    for b in range(B):
        c = rows[b]
        out[b], lse[b] = attention_ref(q[b], c, c[:, :LATENT], scale)
    return out, lse


def tpla_decode_ref(q, rows, G, rope_mode, scale, shard=None):
    """TPLA decode: G latent shards, an independent softmax per shard.

    [ISSUE] "Directions under investigation": every rank attends only over
    the latent columns it holds.  [REVIEW pith_extraction.key_machinery]:
    on each device the softmax is taken over the product of every head's
    query slice with that device's rotated cache slice;
    [REVIEW skeptic_critique]: Eq. 6 applies no scaling to that local
    softmax.
    Shard g's logits use its latent columns plus its rope columns; its
    values are its latent columns only.  Outputs are concatenated in shard
    order (reading 5).

    Returns out [B, H, 512] and lse [B, H, G].  With ``shard = s`` (one-shard
    mode: the work of one TP rank) returns out [B, H, d] and lse [B, H, 1].
    """
    q = np.asarray(q, dtype=np.float64)
    B, H, _ = q.shape
    d = LATENT // G
    shards = range(G) if shard is None else [shard]
    width = LATENT if shard is None else d
    out = np.zeros((B, H, width))
    lse = np.zeros((B, H, len(shards)))
    for b in range(B):
        c = rows[b]
        for k, g in enumerate(shards):
            lat, rope = shard_columns(G, g, rope_mode)
            cols = np.concatenate([lat, rope])
            o, l = attention_ref(q[b][:, cols], c[:, cols], c[:, lat], scale)
            if shard is None:
                out[b][:, lat] = o
            else:
                out[b] = o
            lse[b, :, k] = l
    return out, lse


def gla_decode_ref(q, rows, G, rope_mode, scale):
    """TPLA written as Grouped Latent Attention with G*H heads.

    [REVIEW desk_editor.letter / pith_summary]: TPLA is a special case of
    GLA with replicated heads.  Head (g, h) of the GLA model sees latent group
    g only.  This restatement builds the grouped keys explicitly, evaluates
    all G*H heads in one batched contraction and normalises with SciPy's
    ``logsumexp``, so it shares no softmax code with ``tpla_decode_ref``.
    Returns out [B, H, 512], lse [B, H, G].
    """
    from scipy.special import logsumexp

    q = np.asarray(q, dtype=np.float64)
    B, H, _ = q.shape
    d = LATENT // G
    groups = [shard_columns(G, g, rope_mode) for g in range(G)]
    kdim = d + len(groups[0][1])
    out = np.zeros((B, H, LATENT))
    lse = np.zeros((B, H, G))
    for b in range(B):
        c = rows[b]
        L = c.shape[0]
        # grouped query [G*H, kdim] and grouped keys/values [G, L, *]
        qg = np.stack([q[b][:, np.concatenate(groups[g])] for g in range(G)])
        kg = np.stack([c[:, np.concatenate(groups[g])] for g in range(G)])
        vg = np.stack([c[:, groups[g][0]] for g in range(G)])
        if L == 0:
            lse[b] = -np.inf
            continue
        s = float(scale) * np.einsum("ghk,glk->ghl", qg, kg)  # [G, H, L]
        ls = logsumexp(s, axis=2)  # [G, H]
        w = np.exp(s - ls[..., None])
        o = np.einsum("ghl,glv->ghv", w, vg)  # [G, H, d]
        for g in range(G):
            out[b][:, g * d:(g + 1) * d] = o[g]
            lse[b, :, g] = ls[g]
    return out, lse


def tpla_decode_paged_ref(q, cache, seq_lens, page_table, G, rope_mode,
                          scale, shard=None):
    """``tpla_decode_ref`` on a paged ([num_blocks, 64, 576]) or contiguous
    ([B, Lmax, 576], ``page_table=None``) cache."""
    rows = gather_request_rows(cache, seq_lens, page_table)
    return tpla_decode_ref(q, rows, G, rope_mode, scale, shard)


# ---------------------------------------------------------------------------
# Sequence split + log-sum-exp merge
# ---------------------------------------------------------------------------

def lse_merge_ref(o_parts, lse_parts):
    """Merge attention results of disjoint key chunks.

    [ISSUE] "Directions under investigation": the exact context/sequence
    parallel alternative splits the sequence and merges with the
    flash-attention log-sum-exp rule.  o_parts [S, ..., V] (each chunk's
    normalised output), lse_parts [S, ...].  lse = log sum_k exp(lse_k),
    out = sum_k exp(lse_k - lse) o_k.  Chunks with lse = -inf weigh 0; if
    all are -inf the result is out 0, lse -inf.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    M = lse_parts.max(axis=0)
    finite = np.isfinite(M)
    Ms = np.where(finite, M, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - Ms), 0.0)
    z = w.sum(axis=0)
    lse = np.where(finite, Ms + np.log(np.where(finite, z, 1.0)), -np.inf)
    zz = np.where(finite, z, 1.0)
    out = (w[..., None] * o_parts).sum(axis=0) / zz[..., None]
    out = np.where(finite[..., None], out, 0.0)
    return out, lse


def split_decode_ref(q, rows, G, rope_mode, scale, bounds):
    """TPLA decode with each request's tokens cut at ``bounds`` (a sorted list
    of token offsets starting at 0 and ending at L_b or beyond) and merged
    with ``lse_merge_ref``.  Used to check that the split path is exact."""
    q = np.asarray(q, dtype=np.float64)
    B, H, _ = q.shape
    outs, lses = [], []
    for k in range(len(bounds) - 1):
        chunk = [r[bounds[k]:bounds[k + 1]] for r in rows]
        o, l = tpla_decode_ref(q, chunk, G, rope_mode, scale)
        d = LATENT // G
        # per-shard merge: lay each shard's lse next to its columns
        outs.append(o.reshape(B, H, G, d))
        lses.append(l)
    o, l = lse_merge_ref(np.stack(outs), np.stack(lses))
    return o.reshape(B, H, LATENT), l


# ---------------------------------------------------------------------------
# Orthogonal (Walsh-Hadamard) reparameterisation
# ---------------------------------------------------------------------------

def hadamard_matrix(n: int):
    """Orthonormal Sylvester Hadamard matrix, natural order:
    H[i, j] = (-1)^popcount(i & j) / sqrt(n)  (reading 7).

    [ISSUE] "Directions under investigation" and [ABSTRACT]: an orthogonal
    transform (Hadamard or PCA) applied to the latent before TP slicing.
    """
    if n <= 0 or n & (n - 1):
        raise ValueError("n must be a power of two")
    i = np.arange(n)
    parity = np.zeros((n, n), dtype=np.int64)
    x = i[:, None] & i[None, :]
    while np.any(x):
        parity ^= x & 1
        x = x >> 1
    return np.where(parity == 1, -1.0, 1.0) / math.sqrt(n)


def hadamard_ref(x, dim):
    """Apply the orthonormal Hadamard transform to the first ``dim`` columns
    of every row of ``x`` (rows are the last axis); other columns unchanged."""
    x = np.array(x, dtype=np.float64, copy=True)
    Hm = hadamard_matrix(dim)
    x[..., :dim] = x[..., :dim] @ Hm  # H is symmetric: row-vector form
    return x


# ---------------------------------------------------------------------------
# PCA reparameterisation (the pages' other orthogonal transform)
# ---------------------------------------------------------------------------

def latent_covariance_ref(F):
    """Mean [D] and covariance [D, D] of calibration rows ``F`` [N, D]: the
    mean-centred second moment (1/N) sum (f - m)^T (f - m) (reading 8)."""
    F = np.asarray(F, np.float64)
    if F.ndim != 2 or F.shape[0] == 0:
        raise ValueError("F must be [N, D] with N > 0")
    m = F.mean(axis=0)
    Fc = F - m
    return m, Fc.T @ Fc / F.shape[0]


def pca_basis_ref(F):
    """Principal axes of calibration latents ``F`` [N, D] (reading 8).

    [ABSTRACT] and [ISSUE] "Directions under investigation": an orthogonal
    transform such as PCA is applied before TP slicing.  [REVIEW referee
    report, minor comment on Sec. 4.3.2 / Eq. (25)]: PCA of the collected
    latent features, position features excluded.  [REVIEW pith extraction,
    key machinery]: the orthogonal U is absorbed into the MLA projections.
    The symmetric eigensolver is a library primitive.  Returns
    (lam [D] descending, U [D, D] with the eigenvectors as columns).
    """
    _, C = latent_covariance_ref(F)
    lam, V = np.linalg.eigh(C)
    order = np.argsort(-lam, kind="stable")
    lam, V = lam[order], V[:, order]
    lead = np.argmax(np.abs(V), axis=0)
    sign = np.sign(V[lead, np.arange(V.shape[1])])
    return lam, V * np.where(sign == 0, 1.0, sign)


def pca_calibrate_ref(rows):
    """PCA basis from calibration cache rows [N, 576]: latent columns only,
    the rope part excluded (reading 8)."""
    rows = np.asarray(rows, np.float64)
    return pca_basis_ref(rows[:, :LATENT])


def shard_variance_fractions(lam, G):
    """Each shard's share of the eigenvalue sum over its contiguous index
    range [g d, (g + 1) d), d = len(lam) / G; for G = 2 these are Eq. (25)'s
    alpha and beta with disjoint ranges (reading 9)."""
    lam = np.asarray(lam, np.float64)
    if lam.shape[0] % G:
        raise ValueError("G must divide the dimension")
    d = lam.shape[0] // G
    return np.array([lam[g * d:(g + 1) * d].sum() for g in range(G)]) / lam.sum()


def pca_rotate_ref(x, U, dim=LATENT):
    """x[..., :dim] <- x[..., :dim] U on every row; other columns (rope)
    unchanged.  The same U rotates q's latent part and the cache rows, so the
    global latent logits q c^T are unchanged (U U^T = I)."""
    x = np.array(x, dtype=np.float64, copy=True)
    x[..., :dim] = x[..., :dim] @ np.asarray(U, np.float64)
    return x


def pca_unrotate_ref(out_latent, U):
    """Back from the rotated latent space: out U^T."""
    return np.asarray(out_latent, np.float64) @ np.asarray(U, np.float64).T


def fold_vup_ref(W_uv, U):
    """V-up weights for outputs in the rotated space: W'[h] = U^T W[h], so
    that (out U) W' = out W (the rotation absorbed into the projection)."""
    return np.einsum("ji,hjk->hik", np.asarray(U, np.float64), np.asarray(W_uv, np.float64))


# ---------------------------------------------------------------------------
# Cache append: the latent of a new token, normalised per shard and stored
# ---------------------------------------------------------------------------

def rms_norm_groups_ref(x, groups, eps):
    """RMS normalisation of each of ``groups`` contiguous column blocks of the
    rows of ``x`` (last axis): block / sqrt(mean(block^2) + eps) (reading 10).

    [REVIEW pith_extraction.key_machinery]: Condition 1 asks the shards' RMS
    norms to be proportional to the global norm, i.e. each device normalises
    its own slice of the latent; ``groups = 1`` is the ordinary (global)
    norm of exact MLA.
    """
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    if D % groups:
        raise ValueError("groups must divide the row width")
    d = D // groups
    out = np.empty_like(x)
    for g in range(groups):
        blk = x[..., g * d:(g + 1) * d]
        ms = (blk * blk).mean(axis=-1, keepdims=True)
        out[..., g * d:(g + 1) * d] = blk / np.sqrt(ms + eps)
    return out


def cache_row_ref(kv_new, norm_groups, hadamard, eps):
    """The stored cache row of a new token (reading 10).

    ``kv_new`` [..., 576]: the token's latent before its normalisation
    (columns 0..511) and its rope key (512..575, already position-encoded).
    The latent is optionally rotated by the orthonormal Hadamard matrix
    (the reparameterisation applied before slicing, [ISSUE] "Directions under
    investigation"), then RMS-normalised over ``norm_groups`` contiguous
    shards.  [REVIEW referee_report.significance]: Proposition 1, RMSNorm
    commutes with an orthogonal transform, so with one group rotating before
    or after the norm gives the same row.  The rope part is stored as given.
    """
    a = np.asarray(kv_new, np.float64)
    x = a[..., :LATENT]
    if hadamard:
        x = x @ hadamard_matrix(LATENT)
    return np.concatenate([rms_norm_groups_ref(x, norm_groups, eps), a[..., LATENT:]], axis=-1)


def cache_append_ref(cache, kv_new, positions, page_table, norm_groups, hadamard, eps):
    """A copy of ``cache`` with request b's new row stored at token
    ``positions[b]``: paged, block ``page_table[b][pos // 64]`` row
    ``pos % 64`` of [num_blocks, 64, 576]; contiguous (``page_table=None``),
    row ``pos`` of [B, Lmax, 576].  Nothing else changes."""
    out = np.array(cache, dtype=np.float64, copy=True)
    rows = cache_row_ref(kv_new, norm_groups, hadamard, eps)
    for b, pos in enumerate(np.asarray(positions).tolist()):
        if page_table is None:
            out[b, pos] = rows[b]
        else:
            out[np.asarray(page_table)[b][pos // BLOCK], pos % BLOCK] = rows[b]
    return out


def mla_prefill_ref(q, rows, start, scale):
    """Exact MLA over a request's prompt tokens, causally (reading 11).

    Prompt token i sits at position start + i and attends, with one softmax
    over all 576 values per token as in ``mla_decode_ref``, to the request's
    stored rows 0 .. start + i: the rows cached before the prompt and the
    prompt's own rows up to and including itself.
    q [T, H, 576] (absorbed queries of the prompt tokens); rows
    [>= start + T, 576] (the request's stored rows, in position order).
    Returns out [T, H, 512] and lse [T, H].
    """
    q = np.asarray(q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    T, H, _ = q.shape
    if start < 0 or rows.shape[0] < start + T:
        raise ValueError("rows must hold the prefix and every prompt token")
    out = np.zeros((T, H, LATENT))
    lse = np.zeros((T, H))
    for i in range(T):
        c = rows[:start + i + 1]
        out[i], lse[i] = attention_ref(q[i], c, c[:, :LATENT], scale)
    return out, lse


# ---------------------------------------------------------------------------
# V up-projection combine (stands in for the o_proj all-reduce)
# ---------------------------------------------------------------------------

def vup_ref(out_latent, W_uv):
    """y[b, h, :] = sum_j out[b, h, j] W_uv[h, j, :].

    [ISSUE] "Directions under investigation": shard outputs are combined by
    the existing o_proj all-reduce; with shards laid side by side in latent
    space that sum over shards is the contraction over j (reading 5).
    out_latent [B, H, 512], W_uv [H, 512, Dv] -> y [B, H, Dv].
    """
    return np.einsum("bhj,hjk->bhk", np.asarray(out_latent, np.float64),
                     np.asarray(W_uv, np.float64))


def vup_sharded_ref(out_latent, W_uv, G):
    """The same combine written as the pages describe the deployment: each
    shard's partial product out_g W_uv[h, I_g, :], then a sum over shards
    (the all-reduce)."""
    out_latent = np.asarray(out_latent, np.float64)
    W_uv = np.asarray(W_uv, np.float64)
    d = LATENT // G
    parts = [np.einsum("bhj,hjk->bhk", out_latent[:, :, g * d:(g + 1) * d],
                       W_uv[:, g * d:(g + 1) * d, :]) for g in range(G)]
    return np.sum(parts, axis=0)


# ---------------------------------------------------------------------------
# Diagnostics (informational only; never pass/fail)
# ---------------------------------------------------------------------------

def per_head_cosine(a, b):
    """Cosine similarity per (request, head) of two [B, H, V] outputs.

    [REVIEW skeptic_critique.concrete_test] proposes the per-head cosine of
    the TPLA output against exact MLA as the direct fidelity measurement.
    """
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    num = (a * b).sum(-1)
    den = np.linalg.norm(a, axis=-1) * np.linalg.norm(b, axis=-1)
    return num / np.where(den == 0, 1.0, den)
