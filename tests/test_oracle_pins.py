"""Pins of the fp64 oracle to facts the pages and the mathematics fix.

Every check here is independent of the oracle's own code path: hand-derived
fixtures, closed forms, brute force with scalar loops, a library routine for
the textbook special case, and invariants.  A plausible slip in the oracle (a
dropped mask, a wrong index or sign, a transposed operand, a wrong
normalisation, an inverted label) fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_video_profile_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "masks_small_cases.txt")


# ---------------------------------------------------------------- fixtures

def _read_golden():
    cases, cur, sec = [], None, None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("case"):
            kv = dict(t.split("=") for t in line.split()[1:])
            cur = {k: int(v) for k, v in kv.items()}
            cases.append(cur)
        elif line.startswith("["):
            sec = line.strip("[]")
            cur[sec] = []
        else:
            cur[sec].append(line)
    for c in cases:
        for sec in ("spatial", "temporal", "temporal_token_major"):
            c[sec] = np.array([[ch == "1" for ch in row] for row in c[sec]])
        c["pi"] = np.array([int(t) for t in c["pi"][0].split()])
    return cases


@pytest.mark.parametrize("case", _read_golden(), ids=lambda c: f"N{c['N']}F{c['F']}")
def test_masks_match_hand_derived_fixture(case):
    N, F, a1, a2 = case["N"], case["F"], case["a1"], case["a2"]
    np.testing.assert_array_equal(oracle.spatial_mask(N, F, a1), case["spatial"])
    np.testing.assert_array_equal(oracle.temporal_mask(N, F, a2), case["temporal"])
    np.testing.assert_array_equal(oracle.token_major_index(N, F), case["pi"])
    # permuted temporal mask: entry (x', y') of the token-major view
    pi = oracle.token_major_index(N, F)
    inv = np.argsort(pi)
    mt = oracle.temporal_mask(N, F, a2)
    np.testing.assert_array_equal(mt[np.ix_(inv, inv)], case["temporal_token_major"])
    np.testing.assert_array_equal(oracle.banded_mask(N * F, N, a2), case["temporal_token_major"])


# ------------------------------------------------------------- mask pins

def _masks_by_definition(N, F, a1, a2):
    """Scalar loops over token pairs (i1, j1), (i2, j2) straight from the
    (i, j) definitions."""
    L = N * F
    ms = np.zeros((L, L), dtype=bool)
    mt = np.zeros((L, L), dtype=bool)
    for i1, j1, i2, j2 in itertools.product(range(N), range(F), range(N), range(F)):
        x1, x2 = i1 * F + j1, i2 * F + j2
        ms[x1, x2] = abs(i1 - i2) < a1
        mt[x1, x2] = abs(j1 - j2) < a2
    return ms, mt


@pytest.mark.parametrize("N,F,a1,a2", [(3, 5, 1, 1), (4, 6, 2, 3), (5, 4, 5, 4), (2, 7, 3, 9), (6, 3, 2, 2)])
def test_masks_match_ij_definition(N, F, a1, a2):
    ms, mt = _masks_by_definition(N, F, a1, a2)
    np.testing.assert_array_equal(oracle.spatial_mask(N, F, a1), ms)
    np.testing.assert_array_equal(oracle.temporal_mask(N, F, a2), mt)
    # rows= restriction selects the same rows
    rows = np.array([0, N * F - 1, F // 2 + F])
    rows = rows[rows < N * F]
    np.testing.assert_array_equal(oracle.spatial_mask(N, F, a1, rows), ms[rows])
    np.testing.assert_array_equal(oracle.temporal_mask(N, F, a2, rows), mt[rows])


def _closed_count(n, a):
    # pairs (u, v) in [0, n) with |u - v| < a: the diagonal plus 2 * sum_{t=1}^{a-1} (n - t)
    a = min(a, n)
    return n + 2 * sum(n - t for t in range(1, a))


@pytest.mark.parametrize("N,F,a1,a2", [(4, 64, 1, 4), (8, 256, 2, 16), (5, 7, 5, 7), (3, 11, 2, 20)])
def test_mask_density_closed_form_explicit(N, F, a1, a2):
    ms = oracle.spatial_mask(N, F, a1)
    mt = oracle.temporal_mask(N, F, a2)
    assert ms.sum() == F * F * _closed_count(N, a1)
    assert mt.sum() == N * N * _closed_count(F, a2)
    # the algebraic form n(2a-1) - a(a-1) of the same count (a <= n)
    for n, a in ((N, min(a1, N)), (F, min(a2, F))):
        assert _closed_count(n, a) == n * (2 * a - 1) - a * (a - 1)


@pytest.mark.parametrize("name,sp_density,tp_density", [
    ("tiny", 0.2500, 0.1064), ("small", 0.3438, 0.1174),
    ("cogvideox", 0.3491, 0.2495), ("hunyuan", 0.1460, 0.1498)])
def test_mask_density_large_configs_by_row_counting(name, sp_density, tp_density):
    """Row counts of the oracle's masks (one row per frame for the spatial
    mask, one row per in-frame position for the temporal one; every other row
    is a copy by symmetry) against the closed form and the densities the band
    widths were chosen for."""
    wl = synth.WORKLOADS[name]
    N, F, L = wl.N, wl.F, wl.L
    sp_rows = np.arange(N) * F
    tp_rows = np.arange(F)
    sp = oracle.spatial_mask(N, F, wl.a1, sp_rows).sum() * F
    tp = sum(int(oracle.temporal_mask(N, F, wl.a2, tp_rows[c:c + 64]).sum())
             for c in range(0, F, 64)) * N
    assert sp == F * F * _closed_count(N, wl.a1)
    assert tp == N * N * _closed_count(F, wl.a2)
    assert abs(sp / L ** 2 - sp_density) < 5e-5
    assert abs(tp / L ** 2 - tp_density) < 5e-5


@pytest.mark.parametrize("N,F,a1,a2", [(4, 6, 2, 3), (5, 24, 3, 4), (3, 10, 1, 10), (7, 5, 4, 1)])
def test_spatial_is_block_banded_and_permuted_temporal_is_block_banded(N, F, a1, a2):
    L = N * F
    np.testing.assert_array_equal(oracle.spatial_mask(N, F, a1), oracle.banded_mask(L, F, a1))
    pi = oracle.token_major_index(N, F)
    assert sorted(pi.tolist()) == list(range(L))  # a bijection
    inv = np.argsort(pi)
    mt = oracle.temporal_mask(N, F, a2)
    np.testing.assert_array_equal(mt[np.ix_(inv, inv)], oracle.banded_mask(L, N, a2))


@pytest.mark.parametrize("N,F,a2", [(4, 9, 2), (5, 6, 1), (3, 8, 8)])
def test_temporal_mask_has_2N_minus_1_slashes(N, F, a2):
    """The unmasked pairs fall on exactly 2N-1 slashes, one per frame offset
    k = i1 - i2, each holding the pairs |j1 - j2| < a2 ("Sparse Video-Gen",
    Temporal Head)."""
    mt = oracle.temporal_mask(N, F, a2)
    x1, x2 = np.nonzero(mt)
    k = x1 // F - x2 // F
    assert sorted(set(k.tolist())) == list(range(-(N - 1), N))
    for kk in range(-(N - 1), N):
        assert (k == kk).sum() == (N - abs(kk)) * _closed_count(F, a2)


# ------------------------------------------------------------ attention pins

def _brute_attention(q, k, v, mask, scale):
    """Scalar loops with math.exp: the softmax-weighted average of value rows."""
    R, d = len(q), len(q[0])
    out = []
    for r in range(R):
        scores = []
        for y in range(len(k)):
            if mask is None or mask[r][y]:
                scores.append((y, scale * sum(q[r][c] * k[y][c] for c in range(d))))
        mx = max(s for _, s in scores)
        w = [(y, math.exp(s - mx)) for y, s in scores]
        z = sum(e for _, e in w)
        out.append([sum(e * v[y][c] for y, e in w) / z for c in range(len(v[0]))])
    return np.array(out)


def test_attention_matches_bruteforce_with_masks():
    rng = np.random.default_rng(3)
    N, F, d = 3, 4, 3
    L = N * F
    q, k, v = (rng.standard_normal((L, d)) for _ in range(3))
    v = rng.standard_normal((L, 5))  # value width differs from d: catches a transposed operand
    for mask in (None, oracle.spatial_mask(N, F, 2), oracle.temporal_mask(N, F, 2)):
        got = oracle.attention(q, k, v, mask)
        ref = _brute_attention(q.tolist(), k.tolist(), v.tolist(),
                               None if mask is None else mask.tolist(), 1 / math.sqrt(d))
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_dense_attention_matches_library_sdpa():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((1, 2, 40, 16)) for _ in range(3))
    got = oracle.dense_attention(q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(t) for t in (q, k, v))).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_softmax_invariants():
    rng = np.random.default_rng(7)
    q, k = rng.standard_normal((6, 4)), rng.standard_normal((9, 4))
    mask = rng.random((6, 9)) < 0.5
    mask[:, 0] = True
    p = oracle.attention_probs(q, k, mask)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-14)
    assert np.all(p[~mask] == 0)
    # a per-row constant added to the scores changes nothing: append a column
    # c_r / scale to q and a column of ones to k
    scale = 0.5
    c = rng.standard_normal(6) * 10
    q2 = np.concatenate([q, (c / scale)[:, None]], axis=1)
    k2 = np.concatenate([k, np.ones((9, 1))], axis=1)
    np.testing.assert_allclose(oracle.attention_probs(q2, k2, mask, scale),
                               oracle.attention_probs(q, k, mask, scale), rtol=1e-12, atol=1e-15)


def _rand_qkv(B, H, L, d, seed):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((B, H, L, d)) for _ in range(3))


def test_full_bands_equal_dense():
    N, F, d = 4, 6, 8
    q, k, v = _rand_qkv(1, 2, N * F, d, 11)
    dense = oracle.dense_attention(q, k, v)
    for label in (np.array([[0, 0]]), np.array([[1, 1]])):
        np.testing.assert_allclose(oracle.sparse_attention(q, k, v, label, N, F, N, F), dense,
                                   rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(oracle.sparse_attention_via_layout(q, k, v, label, N, F, N, F),
                                   dense, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("N,F,a1,a2", [(4, 6, 2, 2), (5, 8, 1, 3), (3, 12, 3, 5)])
def test_layout_transformation_is_equivalent(N, F, a1, a2):
    """permute -> block-banded attention -> unpermute equals attention under
    the temporal mask in the original layout (SVG2 explainer, 2.A)."""
    q, k, v = _rand_qkv(1, 2, N * F, 6, 13)
    label = np.array([[0, 1]])
    np.testing.assert_allclose(oracle.sparse_attention_via_layout(q, k, v, label, N, F, a1, a2),
                               oracle.sparse_attention(q, k, v, label, N, F, a1, a2),
                               rtol=1e-12, atol=1e-13)
    x = q[0, 0]
    np.testing.assert_array_equal(oracle.unpermute(oracle.permute(x, N, F), N, F), x)
    # the token (i, j) lands at row j*N + i
    xp = oracle.permute(x, N, F)
    for i, j in itertools.product(range(N), range(F)):
        np.testing.assert_array_equal(xp[j * N + i], x[i * F + j])


def test_rows_subset_matches_full():
    N, F = 3, 8
    q, k, v = _rand_qkv(1, 2, N * F, 4, 17)
    label = np.array([[1, 0]])
    rows = np.array([0, 5, 9, 23])
    full = oracle.sparse_attention(q, k, v, label, N, F, 2, 3)
    part = oracle.sparse_attention(q, k, v, label, N, F, 2, 3, rows=rows)
    np.testing.assert_allclose(part, full[:, :, rows], rtol=1e-13, atol=1e-14)


# ------------------------------------------------------------ profiling pins

def _brute_profile(q, k, v, N, F, a1, a2, rows):
    d = len(q[0])
    sc = 1 / math.sqrt(d)
    ms = [[abs(x // F - y // F) < a1 for y in range(N * F)] for x in rows]
    mt = [[abs(x % F - y % F) < a2 for y in range(N * F)] for x in rows]
    qr = [q[x] for x in rows]
    od = _brute_attention(qr, k, v, None, sc)
    os_ = _brute_attention(qr, k, v, ms, sc)
    ot = _brute_attention(qr, k, v, mt, sc)
    n = len(rows) * len(v[0])
    mse_s = sum((os_[r][c] - od[r][c]) ** 2 for r in range(len(rows)) for c in range(len(v[0]))) / n
    mse_t = sum((ot[r][c] - od[r][c]) ** 2 for r in range(len(rows)) for c in range(len(v[0]))) / n
    return mse_s, mse_t


def test_profile_matches_bruteforce():
    N, F, d = 3, 5, 4
    q, k, v = _rand_qkv(1, 3, N * F, d, 19)
    q[0, 1] *= 3.0  # sharpen one head
    rows = np.array([1, 7, 8, 14])
    mse, label = oracle.profile_heads(q, k, v, N, F, 2, 2, rows)
    for h in range(3):
        ms, mt = _brute_profile(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), N, F, 2, 2, rows)
        np.testing.assert_allclose(mse[0, h], [ms, mt], rtol=1e-10, atol=1e-15)
        assert label[0, h] == (1 if mt < ms else 0)


def test_profile_special_cases():
    N, F = 4, 6
    q, k, v = _rand_qkv(1, 2, N * F, 8, 23)
    rows = np.array([0, 3, 10, 17, 23])
    mse, label = oracle.profile_heads(q, k, v, N, F, N, 2, rows)  # spatial band covers all
    assert np.all(mse[..., 0] == 0) and np.all(mse[..., 1] > 0) and np.all(label == 0)
    mse, label = oracle.profile_heads(q, k, v, N, F, 1, F, rows)  # temporal band covers all
    assert np.all(mse[..., 1] == 0) and np.all(mse[..., 0] > 0) and np.all(label == 1)
    mse, label = oracle.profile_heads(q, k, v, N, F, N, F, rows)  # tie -> spatial
    assert np.all(mse == 0) and np.all(label == 0)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_synthetic_heads_get_their_constructed_labels(name):
    wl = synth.WORKLOADS[name]
    q, k, v = (synth.round_bf16_to_f64(t) for t in synth.make_qkv(wl, seed=0))
    rows = synth.sample_rows(wl.L, wl.S, 0)
    mse, label = oracle.profile_heads(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows)
    np.testing.assert_array_equal(label, synth.head_kinds(wl, 0))
    gap = np.abs(mse[..., 0] - mse[..., 1]) / mse.max(-1)
    assert np.all(gap > 0.2)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_literal_embedding_scale_inverts_the_labels(name):
    """The literal reading of the synthetic heads (embeddings N(0, 1) / sqrt(d))
    gives each head the opposite label: its in-band logit boost, about
    w^2 / sqrt(d), is too small to concentrate the softmax in its band.  This is
    why the default scale is d^(-1/4) (boost about w^2)."""
    wl = synth.WORKLOADS[name]
    q, k, v = (synth.round_bf16_to_f64(t) for t in synth.make_qkv(wl, seed=0, emb_std=wl.d ** -0.5))
    rows = synth.sample_rows(wl.L, wl.S, 0)
    mse, label = oracle.profile_heads(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows)
    np.testing.assert_array_equal(label, 1 - synth.head_kinds(wl, 0))


# ------------------------------------------------------------ block list pin

def _banded_tile_ranges(L, G, a, Bq, Bk, qb):
    q0, q1 = qb * Bq, min(L, (qb + 1) * Bq)
    g_lo, g_hi = q0 // G, (q1 - 1) // G
    lo, hi = max(0, (g_lo - a + 1) * G), min(L, (g_hi + a) * G)
    f_lo, f_hi = max(0, (g_hi - a + 1) * G), min(L, (g_lo + a) * G)
    active = set(range(lo // Bk, -(-hi // Bk)))
    full = {kb for kb in range(-(-L // Bk)) if kb * Bk >= f_lo and min(L, (kb + 1) * Bk) <= f_hi}
    return active, full


@pytest.mark.parametrize("L,G,a,Bq,Bk", [(256, 64, 1, 128, 128), (2048, 8, 16, 128, 128),
                                         (700, 33, 3, 128, 64), (517, 50, 2, 64, 128),
                                         (300, 7, 100, 128, 128), (129, 129, 1, 128, 128)])
def test_block_list_bruteforce_matches_closed_form(L, G, a, Bq, Bk):
    active, full = oracle.block_list(oracle.banded_mask(L, G, a), Bq, Bk)
    for qb in range(active.shape[0]):
        act, ful = _banded_tile_ranges(L, G, a, Bq, Bk, qb)
        assert set(np.nonzero(active[qb])[0].tolist()) == act
        assert set(np.nonzero(full[qb])[0].tolist()) == ful



# ------------------------------------------------------------ mixed-pattern pins

@pytest.mark.parametrize("N,F,W,h,P", [(4, 7, 3, 2, 5), (3, 10, 10, 0, 1), (5, 6, 0, 5, 30)])
def test_mixed_masks_match_definitions(N, F, W, h, P):
    L = N * F
    win = np.zeros((L, L), bool)
    md = np.zeros((L, L), bool)
    for i1, j1, i2, j2 in itertools.product(range(N), range(F), range(N), range(F)):
        x1, x2 = i1 * F + j1, i2 * F + j2
        win[x1, x2] = abs(x1 - x2) <= W
        md[x1, x2] = abs(j1 - j2) <= h
    np.testing.assert_array_equal(oracle.mode_mask(oracle.MODE_DIAGONAL, N, F, W, h, P), win)
    np.testing.assert_array_equal(oracle.mode_mask(oracle.MODE_MULTIDIAG, N, F, W, h, P), md)
    stripe = oracle.mode_mask(oracle.MODE_STRIPE, N, F, W, h, P)
    assert stripe.sum() == L * min(P, L) and np.all(stripe[:, :P]) and not np.any(stripe[:, P:])
    assert oracle.mode_mask(oracle.MODE_FULL, N, F, W, h, P).all()
    assert oracle.mode_mask(oracle.MODE_SKIP, N, F, W, h, P) is None
    # closed forms of the pair counts
    assert win.sum() == L * (2 * min(W, L - 1) + 1) - min(W, L - 1) * (min(W, L - 1) + 1)
    # multi-diagonal on token-major rows is block-banded with G = N, a = h + 1
    inv = np.argsort(oracle.token_major_index(N, F))
    np.testing.assert_array_equal(md[np.ix_(inv, inv)], oracle.banded_mask(L, N, h + 1))


def test_mixed_attention_modes():
    N, F = 4, 6
    rng = np.random.default_rng(31)
    q, k, v = (rng.standard_normal((1, 5, N * F, 3)) for _ in range(3))
    modes = np.array([[0, 1, 2, 3, 4]])
    out = oracle.mixed_attention(q, k, v, modes, N, F, 2, 1, 5)
    np.testing.assert_allclose(out[0, 0], oracle.attention(q[0, 0], k[0, 0], v[0, 0]), rtol=1e-12, atol=1e-13)
    assert np.all(out[0, 1] == 0)  # skipped head: zero output
    # stripe: brute force on the first keys only
    ref = _brute_attention(q[0, 4].tolist(), k[0, 4, :5].tolist(), v[0, 4, :5].tolist(), None, 1 / math.sqrt(3))
    np.testing.assert_allclose(out[0, 4], ref, rtol=1e-12, atol=1e-13)
    # multi-diagonal through the token rearrangement equals the direct mask
    qp, kp, vp = (oracle.permute(t[0, 3], N, F) for t in (q, k, v))
    via = oracle.unpermute(oracle.attention(qp, kp, vp, oracle.banded_mask(N * F, N, 2)), N, F)
    np.testing.assert_allclose(out[0, 3], via, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------ offline mode search pins

@pytest.mark.parametrize("N,F,W,h,P", [(3, 5, 2, 1, 4), (2, 7, 20, 6, 100), (4, 4, 0, 0, 1)])
def test_mode_sparsity_counts(N, F, W, h, P):
    """Sparsity S_i = share of skipped pairs, against closed forms of the three
    masks (window band, |j1 - j2| <= h over all frame pairs, first P keys)."""
    L = N * F
    Wc, a, Pc = min(W, L - 1), min(h + 1, F), min(P, L)
    closed = {
        oracle.MODE_SKIP: 1.0,
        oracle.MODE_DIAGONAL: 1 - (L * (2 * Wc + 1) - Wc * (Wc + 1)) / L**2,
        oracle.MODE_MULTIDIAG: 1 - N * N * (F * (2 * a - 1) - a * (a - 1)) / L**2,
        oracle.MODE_STRIPE: 1 - Pc / L,
    }
    for m, s in closed.items():
        assert oracle.mode_sparsity(m, N, F, W, h, P) == pytest.approx(s, abs=1e-15)


def _one_hot_qkv(N, F, d, target, logit=40.0, seed=0):
    """Keys are unit vectors e_y, query x points at key target(x) with the
    given logit: attention is one-hot on target(x) up to exp(-logit)."""
    L = N * F
    k = np.eye(L, d)[None, None]
    q = np.zeros((1, 1, L, d))
    for x in range(L):
        q[0, 0, x, target(x)] = logit * math.sqrt(d)
    v = np.random.default_rng(seed).standard_normal((1, 1, L, d))
    return q, k, v


@pytest.mark.parametrize("which", ["diagonal", "multidiag", "stripe"])
def test_mode_search_picks_the_exact_mode(which):
    """Attention concentrated on the key a mode keeps: that mode has MSE ~ 0,
    so its loss is lam * (1 - S_i); the others miss the key and pay MSE ~ 1."""
    N, F, d, lam = 2, 3, 8, 0.5
    L = N * F
    target = {"diagonal": lambda x: x,
              "multidiag": lambda x: ((x // F + 1) % N) * F + x % F,
              "stripe": lambda x: 0}[which]
    q, k, v = _one_hot_qkv(N, F, d, target)
    rows = np.arange(L)
    loss, mode = oracle.mode_search(q, k, v, N, F, rows, 0, 0, 1, lam=lam, eps=1.0)
    sp = [oracle.mode_sparsity(m, N, F, 0, 0, 1) for m in oracle.SEARCH_MODES]
    want = {"diagonal": oracle.MODE_DIAGONAL, "multidiag": oracle.MODE_MULTIDIAG, "stripe": oracle.MODE_STRIPE}[which]
    t = oracle.SEARCH_MODES.index(want)
    assert loss[0, 0, t] == pytest.approx(lam * (1 - sp[t]), abs=1e-12)
    assert mode[0, 0] == want
    # the skip loss is the mean square of the dense output (sparsity 1)
    o = np.stack([v[0, 0, target(x)] for x in range(L)])
    assert loss[0, 0, 0] == pytest.approx(np.mean(o**2), rel=1e-12)
    # below every loss the head stays dense
    _, mode = oracle.mode_search(q, k, v, N, F, rows, 0, 0, 1, lam=lam, eps=0.01)
    assert mode[0, 0] == oracle.MODE_FULL


def test_mode_search_constant_values_and_full_bands():
    """V constant over keys: every non-skip mode reproduces the dense output,
    so L_i = lam * (1 - S_i) and the sparsest one wins (a sign error in the
    sparsity term would pick the densest); skip costs mean(c^2).  Bands that
    cover every key give L_i = lam exactly."""
    N, F, d = 3, 4, 5
    L = N * F
    rng = np.random.default_rng(4)
    q, k = (rng.standard_normal((1, 2, L, d)) for _ in range(2))
    c = np.array([3.0, -2.0, 1.0, 0.5, 2.5])
    v = np.broadcast_to(c, (1, 2, L, d)).copy()
    v[0, 1] *= 1e-3  # second head: output so small that skipping is cheapest
    rows = np.array([0, 5, 11])
    loss, mode = oracle.mode_search(q, k, v, N, F, rows, 2, 1, 3, lam=0.5, eps=10.0)
    sp = [oracle.mode_sparsity(m, N, F, 2, 1, 3) for m in oracle.SEARCH_MODES]
    for h in range(2):
        np.testing.assert_allclose(loss[0, h, 1:], 0.5 * (1 - np.array(sp[1:])), atol=1e-12)
    assert loss[0, 0, 0] == pytest.approx(np.mean(c**2), rel=1e-12)
    assert mode[0, 0] == oracle.SEARCH_MODES[1 + int(np.argmax(sp[1:]))]
    assert mode[0, 1] == oracle.MODE_SKIP
    loss, _ = oracle.mode_search(q, k, rng.standard_normal((1, 2, L, d)), N, F, rows, L, F, L, lam=0.7)
    np.testing.assert_allclose(loss[0, :, 1:], 0.7, atol=1e-12)


# ------------------------------------------------------------ SVG2 pins (semantic-aware permutation, top-p)

def _blobs(C, per, d, seed, spread=0.05):
    """C well-separated blobs of `per` rows each, blob c in rows [c per, (c+1) per)."""
    rng = np.random.default_rng(seed)
    centers = rng.standard_normal((C, d)) * 10.0
    x = np.concatenate([centers[c] + spread * rng.standard_normal((per, d)) for c in range(C)])
    return x, np.repeat(np.arange(C), per)


def test_kmeans_recovers_separated_blobs():
    """Rows ordered by blob: the start rows floor(c L / C) are one per blob,
    so one round assigns every row to its blob and the centroids are the
    blob means."""
    x, lab = _blobs(6, 20, 5, 1)
    assign, mu, counts = oracle.kmeans(x, 6, 3)
    np.testing.assert_array_equal(assign, lab)
    np.testing.assert_array_equal(counts, np.full(6, 20))
    for c in range(6):
        np.testing.assert_allclose(mu[c], x[lab == c].mean(0), rtol=0, atol=1e-12)


def test_kmeans_objective_pins():
    """kmeans_objective is the sum of squared row-to-centroid distances: equal
    to a scalar-loop sum, zero when every row sits at its centroid, and the
    hand-computed value of a two-cluster case."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((37, 5))
    mu = rng.standard_normal((4, 5))
    assign = rng.integers(0, 4, size=37)
    loop = sum((x[r][c] - mu[assign[r]][c]) ** 2 for r in range(37) for c in range(5))
    assert abs(oracle.kmeans_objective(x, mu, assign) - loop) <= 1e-12 * loop
    # every row at its centroid: objective 0 exactly
    assert oracle.kmeans_objective(mu[assign], mu, assign) == 0.0
    # rows (0,0), (2,0) with centroid (1,0); rows (0,3), (0,5) with centroid (0,4):
    # 1 + 1 + 1 + 1 = 4
    x2 = np.array([[0.0, 0.0], [2.0, 0.0], [0.0, 3.0], [0.0, 5.0]])
    mu2 = np.array([[1.0, 0.0], [0.0, 4.0]])
    assert oracle.kmeans_objective(x2, mu2, [0, 0, 1, 1]) == 4.0
    # with the assignment swapped: (0,0)-(0,4): 16, (2,0)-(0,4): 4+16, (0,3)-(1,0): 1+9, (0,5)-(1,0): 1+25
    assert oracle.kmeans_objective(x2, mu2, [1, 1, 0, 0]) == 16.0 + 20.0 + 10.0 + 26.0
    # it weighs only the assigned centroid: an unused centroid changes nothing
    mu3 = np.vstack([mu2, [[100.0, 100.0]]])
    assert oracle.kmeans_objective(x2, mu3, [0, 0, 1, 1]) == 4.0


def test_kmeans_objective_never_increases():
    x = np.random.default_rng(2).standard_normal((300, 4))
    prev = np.inf
    for it in range(1, 9):
        assign, mu, _ = oracle.kmeans(x, 7, it)
        obj = oracle.kmeans_objective(x, mu, assign)
        assert obj <= prev + 1e-9
        prev = obj


def test_kmeans_fixed_point_by_brute_force():
    """After convergence every row is at its nearest centroid (scalar-loop
    distances) and every centroid is the mean of its rows (scalar loops)."""
    x = np.random.default_rng(3).standard_normal((120, 3))
    assign, mu, counts = oracle.kmeans(x, 5, 60)
    for r in range(len(x)):
        dist = [sum((x[r][c] - mu[j][c]) ** 2 for c in range(3)) for j in range(5)]
        assert dist[assign[r]] <= min(dist) + 1e-12
    for j in range(5):
        rows = [r for r in range(len(x)) if assign[r] == j]
        assert counts[j] == len(rows)
        for c in range(3):
            assert abs(mu[j][c] - sum(x[r][c] for r in rows) / len(rows)) < 1e-12


def test_kmeans_ties_go_low_and_empty_cluster_keeps_centroid():
    """Duplicate start rows give equal centroids: every row ties between
    them and goes to the lower index, so the higher one is empty and keeps
    its start value."""
    x = np.array([[0.0, 0.0], [0.0, 0.0], [1.0, 0.0], [5.0, 5.0]])
    np.testing.assert_array_equal(oracle.nearest_centroid(x, np.array([[1.0, 1.0], [1.0, 1.0]])), [0, 0, 0, 0])
    x2 = np.array([[3.0, 3.0]] * 4)
    assign, mu, counts = oracle.kmeans(x2, 2, 2)  # starts rows 0 and 2, both (3, 3)
    np.testing.assert_array_equal(assign, [0, 0, 0, 0])
    np.testing.assert_array_equal(counts, [4, 0])
    np.testing.assert_array_equal(mu[1], [3.0, 3.0])


def test_cluster_permutation_is_stable_sort():
    assign = np.random.default_rng(4).integers(0, 6, size=50)
    perm, offsets = oracle.cluster_permutation(assign, 7)
    want = sorted(range(50), key=lambda r: (assign[r], r))
    np.testing.assert_array_equal(perm, want)
    for c in range(7):
        assert list(assign[perm[offsets[c]:offsets[c + 1]]]) == [c] * int((assign == c).sum())
    assert offsets[-1] == 50 and offsets[6] == offsets[7]  # cluster 6 empty


@pytest.mark.parametrize("p", [0.3, 0.7, 0.9, 0.999])
def test_centroid_topp_is_the_minimal_heaviest_prefix(p):
    """The kept set (i) has mass >= p, (ii) loses that by dropping its
    lightest member, (iii) outweighs every cluster it leaves out; with the
    masses recomputed here from n_k exp(scale mu_q . mu_k) by scalar loops."""
    rng = np.random.default_rng(5)
    d = 6
    mu_q, mu_k = rng.standard_normal((4, d)), rng.standard_normal((9, d))
    n_k = rng.integers(0, 30, size=9)
    n_k[3] = 0
    sel = oracle.centroid_topp(mu_q, mu_k, n_k, p)
    s = 1.0 / math.sqrt(d)
    for c in range(4):
        w = [n_k[j] * math.exp(s * sum(mu_q[c][t] * mu_k[j][t] for t in range(d))) for j in range(9)]
        z = sum(w)
        w = [x / z for x in w]
        kept = [j for j in range(9) if sel[c, j]]
        left = [j for j in range(9) if not sel[c, j]]
        assert not sel[c, 3]
        assert sum(w[j] for j in kept) >= p - 1e-12
        assert sum(w[j] for j in kept) - min(w[j] for j in kept) < p
        assert all(w[a] >= w[b] for a in kept for b in left)


def test_centroid_topp_sizes_weight_equal_centroids():
    """Equal centroids: the masses are the size shares (3:1), so p = 0.6
    keeps only the large cluster and p = 0.8 keeps both; p = 1 keeps every
    non-empty cluster."""
    mu_q = np.array([[1.0, 0.0]])
    mu_k = np.array([[0.5, 0.5], [0.5, 0.5], [0.5, 0.5]])
    n_k = np.array([30, 10, 0])
    np.testing.assert_array_equal(oracle.centroid_topp(mu_q, mu_k, n_k, 0.6), [[True, False, False]])
    np.testing.assert_array_equal(oracle.centroid_topp(mu_q, mu_k, n_k, 0.8), [[True, True, False]])
    np.testing.assert_array_equal(oracle.centroid_topp(mu_q, mu_k, n_k, 1.0), [[True, True, False]])


def test_svg2_attention_special_cases_and_permutation():
    rng = np.random.default_rng(6)
    L, d = 40, 4
    q, k, v = (rng.standard_normal((L, d)) for _ in range(3))
    aq, ak = rng.integers(0, 3, L), rng.integers(0, 5, L)
    full = np.ones((3, 5), dtype=bool)
    np.testing.assert_allclose(oracle.svg2_attention_given(q, k, v, aq, ak, full), oracle.attention(q, k, v),
                               rtol=1e-12, atol=1e-13)
    sel = rng.random((3, 5)) < 0.5
    sel[:, 0] = True
    sel[2] = False  # query cluster 2 keeps nothing: its rows are zero
    out = oracle.svg2_attention_given(q, k, v, aq, ak, sel)
    mask = [[bool(sel[aq[x], ak[y]]) for y in range(L)] for x in range(L)]
    keep = [x for x in range(L) if aq[x] != 2]
    ref = _brute_attention(q[keep].tolist(), k.tolist(), v.tolist(), [mask[x] for x in keep], 1 / math.sqrt(d))
    np.testing.assert_allclose(out[keep], ref, rtol=1e-12, atol=1e-13)
    assert np.all(out[aq == 2] == 0)
    via = oracle.svg2_attention_permuted(q, k, v, aq, ak, sel, 3, 5)
    np.testing.assert_allclose(via, out, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- mixed-pattern masks, row attention, SVG2 end to end

@pytest.mark.parametrize("L,W", [(7, 0), (7, 2), (12, 5), (9, 8), (9, 20)])
def test_window_mask_bruteforce_and_count(L, W):
    """|x - y| <= W by scalar loops; count L(2W+1) - W(W+1) while W < L."""
    m = oracle.window_mask(L, W)
    ref = [[abs(x - y) <= W for y in range(L)] for x in range(L)]
    np.testing.assert_array_equal(m, np.array(ref))
    expect = L * L if W >= L - 1 else L * (2 * W + 1) - W * (W + 1)
    assert int(m.sum()) == expect
    rows = [0, L // 2, L - 1]
    np.testing.assert_array_equal(oracle.window_mask(L, W, rows), m[rows])


@pytest.mark.parametrize("L,P", [(8, 0), (8, 3), (8, 8), (8, 11)])
def test_prefix_mask_bruteforce_and_count(L, P):
    """y < P by scalar loops; count L min(P, L); the same for every row."""
    m = oracle.prefix_mask(L, P)
    np.testing.assert_array_equal(m, np.array([[y < P for y in range(L)] for _ in range(L)]))
    assert int(m.sum()) == L * min(P, L)
    np.testing.assert_array_equal(oracle.prefix_mask(L, P, [1, 5]), m[[1, 5]])


def test_head_mask_follows_the_label():
    """Label 0 is the frame band |i1 - i2| < a1, label 1 the position band
    |j1 - j2| < a2 (scalar loops over (i, j))."""
    N, F, a1, a2 = 4, 5, 2, 2
    coords = [(x // F, x % F) for x in range(N * F)]
    sp = [[abs(i1 - i2) < a1 for (i2, _) in coords] for (i1, _) in coords]
    tp = [[abs(j1 - j2) < a2 for (_, j2) in coords] for (_, j1) in coords]
    np.testing.assert_array_equal(oracle.head_mask(oracle.SPATIAL, N, F, a1, a2), np.array(sp))
    np.testing.assert_array_equal(oracle.head_mask(oracle.TEMPORAL, N, F, a1, a2), np.array(tp))


def test_attention_rows_uniform_weights_give_window_means():
    """With q = 0 every kept key has the same weight, so each output row is
    the plain mean of V over its window |x - y| <= W."""
    rng = np.random.default_rng(11)
    L, d, W = 50, 6, 4
    q = np.zeros((L, d))
    k, v = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    rows = np.array([0, 1, 3, 25, 47, 49])
    out = oracle.attention_rows(q, k, v, rows, lambda rr: oracle.window_mask(L, W, rr), chunk=4)
    ref = np.array([v[max(0, x - W):min(L, x + W + 1)].mean(axis=0) for x in rows])
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-14)


def test_svg2_attention_with_p_one_is_dense():
    """Top-p with p = 1 keeps every non-empty key cluster for every query
    cluster, so the whole SVG2 step is dense attention, whatever the
    clustering."""
    rng = np.random.default_rng(12)
    L, d = 60, 8
    q, k, v = (rng.standard_normal((L, d)) for _ in range(3))
    out, aq, ak, sel = oracle.svg2_attention(q, k, v, 4, 6, 3, 1.0)
    probs = np.exp(q @ k.T / math.sqrt(d))
    probs /= probs.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(out, probs @ v, rtol=1e-11, atol=1e-12)
    assert aq.shape == (L,) and ak.shape == (L,) and sel.shape == (4, 6)
