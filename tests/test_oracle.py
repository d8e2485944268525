"""Pins for the CPU float64 oracle: each test checks it against something
other than itself (brute force, closed forms, library routines, invariants
the pages state).  CPU only."""

import json
import math
import os

import numpy as np
import pytest

from oracle import tpla_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
SCALE = np.float64(np.float32(1.0 / math.sqrt(192.0)))


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _rows(B, Ls, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((L, O.WIDTH)) for L in Ls]


# ---------------------------------------------------------------- page figures

def test_page_figures_widths():
    fig = json.load(open(os.path.join(HERE, "golden", "page_figures.json")))
    assert O.WIDTH == fig["values_per_token_mla"]["value"]
    assert O.LATENT == fig["latent_dims"]["value"]
    # one TP=2 rank reads its 256 latent columns plus the replicated rope
    for g in range(2):
        lat, rope = O.shard_columns(2, g, "replicate")
        assert len(lat) + len(rope) == fig["values_per_device_tpla_tp2"]["value"]


def test_shard_columns_partition():
    for G in (1, 2, 4, 8):
        lat_all = np.concatenate([O.shard_columns(G, g)[0] for g in range(G)])
        assert np.array_equal(lat_all, np.arange(512))
        for g in range(G):
            assert np.array_equal(O.shard_columns(G, g, "replicate")[1],
                                  np.arange(512, 576))
    for G in (1, 2, 4):
        rope_all = np.concatenate([O.shard_columns(G, g, "split")[1] for g in range(G)])
        assert np.array_equal(rope_all, np.arange(512, 576))


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("H,L,K,V", [(1, 1, 3, 2), (3, 7, 5, 4), (4, 16, 9, 6)])
def test_attention_matches_bruteforce(H, L, K, V):
    q = _rand((H, K), 1)
    keys = _rand((L, K), 2)
    vals = _rand((L, V), 3)
    o, l = O.attention_ref(q, keys, vals, 0.7)
    ob, lb = O.attention_bruteforce(q.tolist(), keys.tolist(), vals.tolist(), 0.7)
    assert np.allclose(o, np.array(ob), rtol=1e-13, atol=1e-13)
    assert np.allclose(l, np.array(lb), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("G,rope_mode", [(1, "replicate"), (2, "replicate"),
                                         (2, "split"), (4, "split")])
def test_tpla_matches_bruteforce_hardcoded_columns(G, rope_mode):
    """Shard column sets written out here from the definition (not through
    shard_columns), then a scalar-loop softmax per shard."""
    B, H, L = 1, 2, 5
    q = _rand((B, H, O.WIDTH), 11)
    rows = _rows(B, [L], 12)
    out, lse = O.tpla_decode_ref(q, rows, G, rope_mode, SCALE)
    d = 512 // G
    for g in range(G):
        lat = list(range(g * d, g * d + d))
        if rope_mode == "replicate":
            rope = list(range(512, 576))
        else:
            r = 64 // G
            rope = list(range(512 + g * r, 512 + g * r + r))
        cols = lat + rope
        qh = [[q[0, h, j] for j in cols] for h in range(H)]
        keys = [[rows[0][t, j] for j in cols] for t in range(L)]
        vals = [[rows[0][t, j] for j in lat] for t in range(L)]
        ob, lb = O.attention_bruteforce(qh, keys, vals, SCALE)
        assert np.allclose(out[0][:, lat], np.array(ob), rtol=1e-12, atol=1e-12)
        assert np.allclose(lse[0, :, g], np.array(lb), rtol=1e-12, atol=1e-12)


def test_mla_matches_bruteforce():
    B, H, L = 1, 3, 6
    q = _rand((B, H, O.WIDTH), 21)
    rows = _rows(B, [L], 22)
    out, lse = O.mla_decode_ref(q, rows, SCALE)
    keys = rows[0].tolist()
    vals = rows[0][:, :512].tolist()
    ob, lb = O.attention_bruteforce(q[0].tolist(), keys, vals, SCALE)
    assert np.allclose(out[0], np.array(ob), rtol=1e-12, atol=1e-12)
    assert np.allclose(lse[0], np.array(lb), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- invariants

def test_g1_equals_exact_mla():
    """With one shard TPLA is exact MLA (issue, Tests / validation)."""
    B, H = 3, 4
    q = _rand((B, H, O.WIDTH), 31)
    rows = _rows(B, [9, 1, 33], 32)
    o1, l1 = O.tpla_decode_ref(q, rows, 1, "replicate", SCALE)
    om, lm = O.mla_decode_ref(q, rows, SCALE)
    # identical up to the summation order BLAS picks for the gathered columns
    assert np.allclose(o1, om, rtol=1e-13, atol=1e-14)
    assert np.allclose(l1[..., 0], lm, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("G,rope_mode", [(2, "replicate"), (4, "replicate"),
                                         (2, "split"), (4, "split"), (8, "replicate")])
def test_tpla_equals_gla_with_replicated_heads(G, rope_mode):
    """TPLA == GLA with G*H heads (review, desk-editor letter)."""
    B, H = 2, 3
    q = _rand((B, H, O.WIDTH), 41)
    rows = _rows(B, [17, 40], 42)
    ot, lt = O.tpla_decode_ref(q, rows, G, rope_mode, SCALE)
    og, lg = O.gla_decode_ref(q, rows, G, rope_mode, SCALE)
    assert np.allclose(ot, og, rtol=1e-12, atol=1e-13)
    assert np.allclose(lt, lg, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("G,rope_mode", [(1, "replicate"), (2, "replicate"), (4, "split")])
def test_constant_cache_returns_row(G, rope_mode):
    """All cached rows equal r: softmax weights sum to one, so every shard
    returns r's latent slice; lse = scale * q.r + ln L."""
    B, H, L = 2, 5, 13
    q = _rand((B, H, O.WIDTH), 51)
    r = _rand((O.WIDTH,), 52)
    rows = [np.tile(r, (L, 1)) for _ in range(B)]
    out, lse = O.tpla_decode_ref(q, rows, G, rope_mode, SCALE)
    for b in range(B):
        assert np.allclose(out[b], np.tile(r[:512], (H, 1)), rtol=1e-12, atol=1e-12)
        for g in range(G):
            lat, rope = O.shard_columns(G, g, rope_mode)
            cols = np.concatenate([lat, rope])
            expect = SCALE * (q[b][:, cols] @ r[cols]) + math.log(L)
            assert np.allclose(lse[b, :, g], expect, rtol=1e-12, atol=1e-12)


def test_zero_query_gives_mean_and_log_len():
    B, H, G = 2, 3, 2
    q = np.zeros((B, H, O.WIDTH))
    rows = _rows(B, [7, 20], 61)
    out, lse = O.tpla_decode_ref(q, rows, G, "replicate", SCALE)
    for b in range(B):
        mean = rows[b][:, :512].mean(axis=0)
        assert np.allclose(out[b], np.tile(mean, (H, 1)), rtol=1e-12, atol=1e-13)
        assert np.allclose(lse[b], math.log(rows[b].shape[0]), rtol=0, atol=1e-13)


def test_empty_request():
    q = _rand((2, 3, O.WIDTH), 71)
    rows = _rows(2, [0, 4], 72)
    out, lse = O.tpla_decode_ref(q, rows, 2, "replicate", SCALE)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


def test_one_shard_mode_is_a_slice():
    B, H, G = 2, 4, 4
    q = _rand((B, H, O.WIDTH), 81)
    rows = _rows(B, [30, 5], 82)
    full, lfull = O.tpla_decode_ref(q, rows, G, "split", SCALE)
    for s in range(G):
        one, l1 = O.tpla_decode_ref(q, rows, G, "split", SCALE, shard=s)
        assert one.shape == (B, H, 512 // G)
        assert np.array_equal(one, full[:, :, s * 128:(s + 1) * 128])
        assert np.array_equal(l1[..., 0], lfull[..., s])


def test_softmax_shift_invariance():
    """Adding a constant to every logit of a shard (here: via a rope column
    that is constant over tokens) leaves the output unchanged and shifts lse
    by exactly that constant."""
    B, H, L = 1, 2, 9
    q = _rand((B, H, O.WIDTH), 91)
    rows = _rows(B, [L], 92)
    base_rows = [rows[0].copy()]
    base_rows[0][:, 512:] = 0.0
    shifted = [base_rows[0].copy()]
    shifted[0][:, 512] = 3.0
    o0, l0 = O.tpla_decode_ref(q, base_rows, 2, "replicate", SCALE)
    o1, l1 = O.tpla_decode_ref(q, shifted, 2, "replicate", SCALE)
    assert np.allclose(o0, o1, rtol=1e-12, atol=1e-13)
    assert np.allclose(l1 - l0, SCALE * 3.0 * q[0][:, 512][:, None], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- paging

def test_paged_equals_contiguous():
    rng = np.random.default_rng(101)
    B, H, Ls = 3, 2, [70, 1, 128]
    cont = rng.standard_normal((B, 128, O.WIDTH))
    pages = [(L + 63) // 64 for L in Ls]
    nb = sum(pages) + 2
    perm = rng.permutation(nb)
    cache = rng.standard_normal((nb, 64, O.WIDTH))
    pt = np.zeros((B, 2), dtype=np.int64)
    off = 0
    for b in range(B):
        for p in range(pages[b]):
            blk = perm[off + p]
            pt[b, p] = blk
            cache[blk] = cont[b, p * 64:(p + 1) * 64]
        off += pages[b]
    q = rng.standard_normal((B, H, O.WIDTH))
    a = O.tpla_decode_paged_ref(q, cache, Ls, pt, 2, "replicate", SCALE)
    c = O.tpla_decode_paged_ref(q, cont, Ls, None, 2, "replicate", SCALE)
    assert np.array_equal(a[0], c[0]) and np.array_equal(a[1], c[1])


# ---------------------------------------------------------------- split + merge

@pytest.mark.parametrize("bounds", [[0, 5, 40], [0, 0, 13, 13, 40], [0, 1, 2, 3, 40],
                                    [0, 40, 64]])
def test_split_merge_equals_unsplit(bounds):
    B, H, G = 2, 3, 2
    q = _rand((B, H, O.WIDTH), 111)
    rows = _rows(B, [40, 17], 112)
    os_, ls_ = O.split_decode_ref(q, rows, G, "replicate", SCALE, bounds)
    ou, lu = O.tpla_decode_ref(q, rows, G, "replicate", SCALE)
    assert np.allclose(os_, ou, rtol=1e-12, atol=1e-13)
    assert np.allclose(ls_, lu, rtol=1e-12, atol=1e-12)


def test_lse_merge_closed_form():
    # two chunks with lse 0 and ln 3: weights 1/4 and 3/4
    o = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])
    l = np.array([[0.0], [math.log(3.0)]])
    out, lse = O.lse_merge_ref(o, l)
    assert np.allclose(out, [[0.25, 0.75]])
    assert np.allclose(lse, [math.log(4.0)])
    # all-empty chunks -> zero output, -inf lse
    out, lse = O.lse_merge_ref(o, np.full((2, 1), -np.inf))
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    # one empty chunk contributes nothing
    out, lse = O.lse_merge_ref(o, np.array([[-np.inf], [0.5]]))
    assert np.allclose(out, [[0.0, 1.0]]) and np.allclose(lse, [0.5])


# ---------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("n", [1, 2, 8, 64, 512])
def test_hadamard_matches_scipy_and_is_involution(n):
    from scipy.linalg import hadamard
    Hm = O.hadamard_matrix(n)
    assert np.allclose(Hm, hadamard(n) / math.sqrt(n), rtol=0, atol=1e-15)
    assert np.allclose(Hm @ Hm, np.eye(n), atol=1e-12)
    e0 = np.zeros(n)
    e0[0] = 1.0
    assert np.allclose(Hm @ e0, np.full(n, 1 / math.sqrt(n)))


def test_hadamard_kron_recursion():
    h2 = np.array([[1.0, 1.0], [1.0, -1.0]])
    M = np.array([[1.0]])
    for _ in range(9):
        M = np.kron(M, h2)
    assert np.allclose(O.hadamard_matrix(512), M / math.sqrt(512), atol=1e-15)


def test_hadamard_ref_leaves_rope_and_preserves_norm():
    x = _rand((5, O.WIDTH), 121)
    y = O.hadamard_ref(x, 512)
    assert np.array_equal(y[:, 512:], x[:, 512:])
    assert np.allclose(np.linalg.norm(y[:, :512], axis=1), np.linalg.norm(x[:, :512], axis=1))
    assert np.allclose(O.hadamard_ref(y, 512), x, atol=1e-12)


def test_hadamard_invariance_for_g1():
    """Orthogonal U absorbed into q and the cache leaves exact MLA unchanged
    after un-rotating the latent output (U U^T = I)."""
    B, H = 2, 3
    q = _rand((B, H, O.WIDTH), 131)
    rows = _rows(B, [25, 64], 132)
    o, l = O.tpla_decode_ref(q, rows, 1, "replicate", SCALE)
    qr = O.hadamard_ref(q, 512)
    rr = [O.hadamard_ref(r, 512) for r in rows]
    o2, l2 = O.tpla_decode_ref(qr, rr, 1, "replicate", SCALE)
    o2 = O.hadamard_ref(o2, 512)
    assert np.allclose(o, o2, atol=1e-12)
    assert np.allclose(l, l2, atol=1e-12)


def test_hadamard_changes_tpla_g2():
    """For G>1 the rotation is not absorbed exactly (the per-shard softmax is
    an approximation): the rotated result differs from the unrotated one."""
    B, H = 1, 2
    q = _rand((B, H, O.WIDTH), 141)
    rows = _rows(B, [30], 142)
    o, _ = O.tpla_decode_ref(q, rows, 2, "replicate", SCALE)
    o2, _ = O.tpla_decode_ref(O.hadamard_ref(q, 512), [O.hadamard_ref(rows[0], 512)],
                              2, "replicate", SCALE)
    assert not np.allclose(o, O.hadamard_ref(o2, 512), atol=1e-6)


# ---------------------------------------------------------------- PCA

def _design(N, D):
    """N x D of +-1 whose columns are zero-mean and mutually orthogonal
    (Z^T Z = N I): non-constant Walsh columns from scipy's Hadamard."""
    from scipy.linalg import hadamard
    return hadamard(N).astype(np.float64)[:, 1:D + 1]


def _planted(offset=1.5):
    """Calibration rows with a known covariance R diag(s^2) R^T (plus a
    constant offset that centring must remove), and the basis the pages'
    PCA must return: R's columns by descending s^2.  R is four plane
    rotations by angles below 45 degrees, so each column's largest entry is
    already positive."""
    D = 8
    R = np.zeros((D, D))
    for k, th in enumerate([0.3, 0.5, 0.1, 0.7]):
        c, s_ = math.cos(th), math.sin(th)
        R[2 * k:2 * k + 2, 2 * k:2 * k + 2] = [[c, -s_], [s_, c]]
    var = np.array([5.0, 0.5, 3.0, 7.0, 1.0, 2.0, 9.0, 4.0])
    F = (_design(64, D) * np.sqrt(var)) @ R.T + offset
    order = [6, 3, 0, 7, 2, 5, 4, 1]
    return F, var[order], R[:, order]


def _matches_planted(basis_fn):
    F, lam_x, U_x = _planted()
    lam, U = basis_fn(F)
    return np.allclose(lam, lam_x, atol=1e-12) and np.allclose(U, U_x, atol=1e-12)


def test_pca_recovers_planted_eigenpairs():
    assert _matches_planted(O.pca_basis_ref)
    F, _, _ = _planted()
    lam, U = O.pca_basis_ref(F)
    assert np.allclose(U.T @ U, np.eye(8), atol=1e-13)


def test_covariance_of_planted_rows():
    """The planted rows' mean is the offset and their covariance is
    R diag(var) R^T, whatever the offset."""
    for off in (0.0, 1.5, -40.0):
        F, lam_x, U_x = _planted(off)
        m, C = O.latent_covariance_ref(F)
        assert np.allclose(m, off, atol=1e-12)
        assert np.allclose(C, U_x @ np.diag(lam_x) @ U_x.T, atol=1e-11)


def test_pca_sign_rule_on_a_tie():
    """45-degree axes: entries tie in magnitude, so the first is made
    positive: (1, 1)/sqrt2 for the larger variance, (1, -1)/sqrt2 next."""
    Z = _design(16, 2)
    F = (Z * [2.0, 1.0]) @ (np.array([[1.0, -1.0], [1.0, 1.0]]) / math.sqrt(2)).T
    lam, U = O.pca_basis_ref(F)
    assert np.allclose(lam, [4.0, 1.0], atol=1e-13)
    assert np.allclose(U, np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2), atol=1e-13)


def test_pca_fractions_of_the_decayed_cache_closed_form():
    """Uncorrelated latent channels with standard deviation exp(-j/128), the
    workloads' decay, stored in a scrambled channel order: PCA sorts them
    back (U is the inverse permutation), lam_j = exp(-j/64), and shard g of G
    holds r^(g d) (1 - r^d) / (1 - r^512) of the sum, r = exp(-1/64); at G = 2
    alpha = 1 / (1 + e^-4) and alpha + beta = 1."""
    D = 512
    s = np.exp(-np.arange(D) / 128.0)
    perm = np.random.default_rng(3).permutation(D)
    F = (_design(1024, D) * s)[:, perm]
    lam, U = O.pca_basis_ref(F)
    assert np.allclose(lam, s ** 2, rtol=1e-10, atol=0)
    assert np.allclose(U, np.eye(D)[:, np.argsort(perm)], atol=1e-10)
    a, b = O.shard_variance_fractions(lam, 2)
    assert abs(a - 1.0 / (1.0 + math.exp(-4.0))) < 1e-12
    assert abs(a + b - 1.0) < 1e-14
    r = math.exp(-1.0 / 64.0)
    for G in (4, 8):
        d = D // G
        want = [r ** (g * d) * (1 - r ** d) / (1 - r ** D) for g in range(G)]
        assert np.allclose(O.shard_variance_fractions(lam, G), want, rtol=1e-10, atol=0)


def test_pca_isotropic_shares_are_equal():
    lam, _ = O.pca_basis_ref(_design(64, 16) * 3.0)
    assert np.allclose(lam, 9.0, atol=1e-12)
    for G in (1, 2, 4, 8):
        assert np.allclose(O.shard_variance_fractions(lam, G), 1.0 / G, atol=1e-14)


def test_pca_leading_axis_matches_power_iteration():
    """Power iteration on the centred rows, an algorithm independent of the
    library eigensolver, finds the same leading axis and eigenvalue."""
    rng = np.random.default_rng(11)
    N, D = 400, 16
    F = rng.standard_normal((N, D)) @ np.diag(np.linspace(3.0, 0.5, D)) + 2.0
    lam, U = O.pca_basis_ref(F)
    Fc = F - F.mean(axis=0)
    v = np.ones(D)
    for _ in range(3000):
        v = Fc.T @ (Fc @ v)
        v /= np.linalg.norm(v)
    v = v if v[np.argmax(np.abs(v))] > 0 else -v
    assert np.allclose(U[:, 0], v, atol=1e-8)
    assert abs(lam[0] - v @ (Fc.T @ (Fc @ v)) / N) < 1e-10


def test_pca_calibration_excludes_rope():
    """The basis comes from the latent columns alone: rope columns with a
    large, correlated variance change nothing."""
    rng = np.random.default_rng(17)
    lat = rng.standard_normal((300, 512)) * np.exp(-np.arange(512) / 128.0)
    rope = 50.0 * lat[:, :64] + rng.standard_normal((300, 64))
    lam, U = O.pca_calibrate_ref(np.concatenate([lat, rope], axis=1))
    lam2, U2 = O.pca_basis_ref(lat)
    assert U.shape == (512, 512)
    assert np.array_equal(lam, lam2) and np.array_equal(U, U2)


def test_pca_rotation_invariance_for_g1_and_fold():
    """U absorbed into q and the cache leaves exact MLA unchanged after the
    output is rotated back, and folding U^T into W_uv gives the same y."""
    rng = np.random.default_rng(19)
    _, U = O.pca_basis_ref(rng.standard_normal((700, 512)) * np.exp(-np.arange(512) / 128.0))
    q = _rand((2, 3, O.WIDTH), 181)
    rows = _rows(2, [40, 65], 182)
    o, l = O.tpla_decode_ref(q, rows, 1, "replicate", SCALE)
    qr = O.pca_rotate_ref(q, U)
    rr = [O.pca_rotate_ref(r, U) for r in rows]
    assert np.array_equal(qr[..., 512:], q[..., 512:])
    o2, l2 = O.tpla_decode_ref(qr, rr, 1, "replicate", SCALE)
    assert np.allclose(O.pca_unrotate_ref(o2, U), o, atol=1e-12)
    assert np.allclose(l2, l, atol=1e-12)
    W = _rand((3, 512, 16), 183)
    assert np.allclose(O.vup_ref(o2, O.fold_vup_ref(W, U)), O.vup_ref(o, W), atol=1e-10)
    # for G = 2 the rotation is not absorbed exactly (shard-local softmax)
    o3, _ = O.tpla_decode_ref(qr, rr, 2, "replicate", SCALE)
    o4, _ = O.tpla_decode_ref(q, rows, 2, "replicate", SCALE)
    assert not np.allclose(O.pca_unrotate_ref(o3, U), o4, atol=1e-6)


def test_pca_pins_catch_planted_mistakes():
    def ascending(F):
        lam, U = O.pca_basis_ref(F)
        return lam[::-1], U[:, ::-1]

    def uncentred(F):
        F = np.asarray(F, np.float64)
        lam, V = np.linalg.eigh(F.T @ F / F.shape[0])
        o = np.argsort(-lam)
        V = V[:, o]
        return lam[o], V * np.sign(V[np.argmax(np.abs(V), axis=0), np.arange(V.shape[1])])

    def transposed(F):
        lam, U = O.pca_basis_ref(F)
        return lam, U.T

    for bad in (ascending, uncentred, transposed):
        assert not _matches_planted(bad)


# ---------------------------------------------------------------- combine

@pytest.mark.parametrize("G", [1, 2, 4])
def test_vup_concat_equals_sum_over_shards(G):
    out = _rand((3, 4, 512), 151)
    W = _rand((4, 512, 128), 152)
    assert np.allclose(O.vup_ref(out, W), O.vup_sharded_ref(out, W, G), atol=1e-10)


def test_vup_hadamard_fold_and_bruteforce():
    out = _rand((2, 2, 512), 161)
    W = _rand((2, 512, 8), 162)
    Hm = O.hadamard_matrix(512)
    W_folded = np.einsum("ij,hjk->hik", Hm, W)
    assert np.allclose(O.vup_ref(O.hadamard_ref(out, 512), W), O.vup_ref(out, W_folded), atol=1e-10)
    y = O.vup_ref(out, W)
    for b in range(2):
        for h in range(2):
            for k in range(8):
                assert abs(y[b, h, k] - sum(out[b, h, j] * W[h, j, k] for j in range(512))) < 1e-10


# ---------------------------------------------------------------- planted mistakes

def test_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in a copy of the oracle's primitive and check
    that an independent pin fails for each."""
    B, H, L = 1, 2, 6
    q = _rand((B, H, O.WIDTH), 171)
    rows = _rows(B, [L], 172)
    keys = rows[0].tolist()
    vals = rows[0][:, :512].tolist()
    ob, lb = O.attention_bruteforce(q[0].tolist(), keys, vals, SCALE)
    good = O.attention_ref

    def no_scale(qh, k, v, s):
        return good(qh, k, v, 1.0)

    def dropped_rope(qh, k, v, s):
        kk = np.array(k, copy=True)
        kk[:, 512:] = 0.0
        return good(qh, kk, v, s)

    def wrong_sign(qh, k, v, s):
        return good(qh, k, v, -s)

    for bad in (no_scale, dropped_rope, wrong_sign):
        monkeypatch.setattr(O, "attention_ref", bad)
        out, lse = O.mla_decode_ref(q, rows, SCALE)
        assert not np.allclose(out[0], np.array(ob), atol=1e-9)
    monkeypatch.setattr(O, "attention_ref", good)


def test_per_head_cosine_hand_computed():
    """The referee's fidelity measure (per-head cosine of two outputs), pinned
    on rows whose cosines are known by hand: parallel (different lengths),
    orthogonal, antiparallel, a 3-4-5 pair, a known angle, and a zero row
    (defined as 0).  Each (request, head) is reduced over the last axis only."""
    a = np.zeros((2, 3, 4))
    b = np.zeros((2, 3, 4))
    a[0, 0, :3], b[0, 0, :3] = [1, 2, 2], [2, 4, 4]          # parallel: 1
    a[0, 1, :3], b[0, 1, :3] = [1, 0, 0], [0, 3, 0]          # orthogonal: 0
    a[0, 2, :2], b[0, 2, :2] = [1, -1], [-2, 2]              # antiparallel: -1
    a[1, 0, :2], b[1, 0, :2] = [3, 4], [8, 6]                # 48 / (5 * 10)
    t = 0.3
    a[1, 1, 2:], b[1, 1, 2:] = [math.cos(t), math.sin(t)], [5, 0]  # angle t
    a[1, 2, :], b[1, 2, :] = [0, 0, 0, 0], [1, 1, 1, 1]      # zero row: 0
    want = np.array([[1.0, 0.0, -1.0], [0.96, math.cos(t), 0.0]])
    got = O.per_head_cosine(a, b)
    assert got.shape == (2, 3)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    # symmetric, and invariant under positive scaling of either argument
    np.testing.assert_allclose(O.per_head_cosine(b, a), want, rtol=0, atol=1e-15)
    np.testing.assert_allclose(O.per_head_cosine(7.0 * a, 0.5 * b), want, rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------
# Cache append: per-shard RMS normalisation (Condition 1 / Proposition 1)
# ---------------------------------------------------------------------------

def _cache_row_bruteforce(a, groups, hadamard, eps):
    """Scalar-loop restatement on Python floats: Sylvester entries from the
    popcount rule, sums of squares and square roots by hand."""
    D = 512
    x = [float(v) for v in a[:D]]
    if hadamard:
        y = []
        for j in range(D):
            acc = 0.0
            for i in range(D):
                sign = -1.0 if bin(i & j).count("1") % 2 else 1.0
                acc += x[i] * sign
            y.append(acc / math.sqrt(D))
        x = y
    d = D // groups
    out = []
    for g in range(groups):
        blk = x[g * d:(g + 1) * d]
        ms = sum(v * v for v in blk) / d
        out += [v / math.sqrt(ms + eps) for v in blk]
    return out + [float(v) for v in a[D:]]


@pytest.mark.parametrize("groups,hadamard", [(1, False), (2, False), (4, True), (8, True)])
def test_cache_row_matches_bruteforce(groups, hadamard):
    a = np.random.default_rng(groups).standard_normal((2, 576)) * 3.0
    got = O.cache_row_ref(a, groups, hadamard, 1e-6)
    for b in range(2):
        want = _cache_row_bruteforce(a[b], groups, hadamard, 1e-6)
        np.testing.assert_allclose(got[b], want, rtol=1e-12, atol=1e-12)


def test_proposition1_rmsnorm_commutes_with_hadamard():
    """With one group, normalising then rotating equals rotating then
    normalising: the orthogonal H keeps the RMS of a row."""
    a = np.random.default_rng(3).standard_normal((5, 576)) * np.exp(-np.arange(576) / 128)
    rot_first = O.cache_row_ref(a, 1, True, 1e-6)
    norm_first = O.hadamard_ref(O.cache_row_ref(a, 1, False, 1e-6), 512)
    np.testing.assert_allclose(rot_first, norm_first, rtol=0, atol=1e-12)
    # with several groups it does not hold in general (the shards' energies differ)
    g2 = O.hadamard_ref(O.cache_row_ref(a, 2, False, 1e-6), 512)
    assert np.abs(O.cache_row_ref(a, 2, True, 1e-6) - g2).max() > 1e-3


def test_condition1_spike_closed_forms():
    """A latent concentrated on one channel: after the Hadamard rotation every
    entry is +-1/sqrt(512), so every shard has the global RMS and the stored
    row is the sign pattern for any number of groups (Condition 1 exact).
    Without the rotation only the shard holding the channel is non-zero, at
    sqrt(d) (d = 512 / groups), and the other shards stay 0."""
    k, eps = 300, 0.0
    a = np.zeros(576)
    a[k] = 2.5
    a[512:] = np.arange(64) * 0.5
    H = O.hadamard_matrix(512)
    for groups in (1, 2, 4, 8):
        row = O.cache_row_ref(a, groups, True, eps)
        np.testing.assert_allclose(row[:512], np.sign(H[k]), rtol=0, atol=1e-12)
        np.testing.assert_array_equal(row[512:], a[512:])
        d = 512 // groups
        plain = O.cache_row_ref(a, groups, False, 1e-30)
        want = np.zeros(512)
        want[k] = math.sqrt(d)
        np.testing.assert_allclose(plain[:512], want, rtol=1e-12, atol=1e-12)


def test_cache_row_groups_have_unit_rms():
    a = np.random.default_rng(4).standard_normal((3, 576)) * 0.01
    eps = 1e-5
    for groups in (1, 2, 4):
        d = 512 // groups
        x = O.hadamard_ref(a, 512)[:, :512]
        row = O.cache_row_ref(a, groups, True, eps)
        for g in range(groups):
            ms = (x[:, g * d:(g + 1) * d] ** 2).mean(axis=1)
            got = (row[:, g * d:(g + 1) * d] ** 2).mean(axis=1)
            np.testing.assert_allclose(got, ms / (ms + eps), rtol=1e-12)


def test_cache_append_placement_paged_and_contiguous():
    rng = np.random.default_rng(5)
    B, pages = 3, 3
    cache = rng.standard_normal((8, 64, 576))
    pt = np.array([[4, 1, 7], [0, 2, 3], [6, 5, 1]])
    pos = np.array([130, 0, 63])
    new = rng.standard_normal((B, 576))
    got = O.cache_append_ref(cache, new, pos, pt, 2, True, 1e-6)
    rows = O.cache_row_ref(new, 2, True, 1e-6)
    want = cache.copy()
    for b in range(B):
        want[pt[b][pos[b] // 64], pos[b] % 64] = rows[b]
    np.testing.assert_array_equal(got, want)
    assert np.count_nonzero(np.any(got != cache, axis=-1)) == B  # nothing else changed
    # the same rows land at the same tokens of a contiguous cache
    contig = np.stack([cache[pt[b]].reshape(pages * 64, 576) for b in range(B)])
    got_c = O.cache_append_ref(contig, new, pos, None, 2, True, 1e-6)
    for b in range(B):
        np.testing.assert_array_equal(got_c[b].reshape(pages, 64, 576), got[pt[b]])


def test_cache_append_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in the oracle's normaliser; the brute-force
    and closed-form pins must fail on each."""
    good = O.rms_norm_groups_ref
    a = np.random.default_rng(6).standard_normal(576)

    def norm_over_width(x, groups, eps):  # one norm over all columns
        return good(x, 1, eps)

    def no_mean(x, groups, eps):  # sum of squares instead of the mean
        d = x.shape[-1] // groups
        return good(x, groups, eps) / math.sqrt(d)

    def interleaved(x, groups, eps):  # shards as strided columns
        x = np.asarray(x, np.float64)
        out = np.empty_like(x)
        for g in range(groups):
            blk = x[..., g::groups]
            out[..., g::groups] = blk / np.sqrt((blk * blk).mean(axis=-1, keepdims=True) + eps)
        return out

    for bad in (norm_over_width, no_mean, interleaved):
        monkeypatch.setattr(O, "rms_norm_groups_ref", bad)
        got = O.cache_row_ref(a, 4, False, 1e-6)
        want = _cache_row_bruteforce(a, 4, False, 1e-6)
        assert np.abs(got - np.asarray(want)).max() > 1e-3, bad.__name__
    monkeypatch.setattr(O, "rms_norm_groups_ref", good)


# ---------------------------------------------------------------- prefill (exact MLA, causal)

def _masked_prefill(q, rows, start, scale):
    """Causal attention written as one score matrix over all stored rows with
    the positions after each query masked to -inf (the mask form, not the
    prefix slices the oracle takes)."""
    T, H, _ = q.shape
    n = start + T
    out = np.zeros((T, H, O.LATENT))
    lse = np.zeros((T, H))
    for i in range(T):
        for h in range(H):
            s = np.array([scale * math.fsum(float(a) * float(b) for a, b in zip(q[i, h], rows[t]))
                          for t in range(n)])
            s[np.arange(n) > start + i] = -np.inf
            m = s.max()
            w = np.exp(s - m)
            z = math.fsum(w)
            out[i, h] = (w[:, None] * rows[:n, :O.LATENT]).sum(0) / z
            lse[i, h] = m + math.log(z)
    return out, lse


@pytest.mark.parametrize("start", [0, 3])
def test_prefill_matches_masked_bruteforce(start):
    T, H = 4, 2
    q = _rand((T, H, O.WIDTH), 40 + start)
    rows = _rand((start + T, O.WIDTH), 50 + start)
    got_o, got_l = O.mla_prefill_ref(q, rows, start, SCALE)
    want_o, want_l = _masked_prefill(q, rows, start, SCALE)
    np.testing.assert_allclose(got_o, want_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got_l, want_l, rtol=1e-12, atol=1e-12)


def test_prefill_first_token_closed_form():
    """With nothing cached, prompt token 0 sees only its own row: the output
    is that row's latent and lse its own score."""
    q = _rand((3, 4, O.WIDTH), 61)
    rows = _rand((3, O.WIDTH), 62)
    out, lse = O.mla_prefill_ref(q, rows, 0, SCALE)
    np.testing.assert_allclose(out[0], np.broadcast_to(rows[0, :O.LATENT], (4, O.LATENT)),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse[0], SCALE * (q[0] @ rows[0]), rtol=1e-12, atol=1e-12)


def test_prefill_last_token_is_a_decode_and_causal():
    start, T, H = 5, 6, 3
    q = _rand((T, H, O.WIDTH), 63)
    rows = _rand((start + T, O.WIDTH), 64)
    out, lse = O.mla_prefill_ref(q, rows, start, SCALE)
    # the last prompt token attends to the whole request: one decode step
    do, dl = O.mla_decode_ref(q[-1:], [rows], SCALE)
    np.testing.assert_allclose(out[-1], do[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse[-1], dl[0], rtol=1e-12, atol=1e-12)
    # rows after position start + i never reach token i; they do reach later ones
    other = rows.copy()
    other[start + 3:] += 1.0
    out2, _ = O.mla_prefill_ref(q, other, start, SCALE)
    np.testing.assert_array_equal(out2[:3], out[:3])
    assert np.abs(out2[3:] - out[3:]).max() > 1e-3


def test_prefill_pins_catch_planted_mistakes(monkeypatch):
    """An off-by-one prefix (token i seeing only rows before it) fails the
    closed form and the masked brute force."""
    good = O.attention_ref
    q = _rand((3, 2, O.WIDTH), 65)
    rows = _rand((3, O.WIDTH), 66)

    def shifted(qh, keys, values, scale):  # drops the token's own row
        return good(qh, keys[:-1], values[:-1], scale)

    monkeypatch.setattr(O, "attention_ref", shifted)
    out, _ = O.mla_prefill_ref(q, rows, 0, SCALE)
    assert not np.allclose(out[0], rows[0, :O.LATENT])
    want, _ = _masked_prefill(q, rows, 0, SCALE)
    assert not np.allclose(out, want)
