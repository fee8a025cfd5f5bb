"""GPU parity: every CUDA entry point against the fp64 oracle.

Tolerances (outputs compared element by element with the oracle run on the
very same, already-rounded inputs):
  bf16 inputs, fp32 accumulation, bf16 output: max-abs 2e-2 and relative L2
      1e-2.
  fp32 inputs and outputs (CUDA-core fp32 arithmetic): max-abs 1e-4 and
      relative L2 1e-5.  fp32 accumulation over at most a few thousand
      terms of magnitude <= 1 stays well inside these.
Data movement (permute / unpermute) and labels are bit-exact.  Labels are
compared on heads whose oracle MSE gap exceeds 1e-3 relative.  Profiling MSEs
(and the MSE parts of the mode-search losses) are compared with the oracle's
value head by head, within a bound derived from the kernels' own rounding
(one bf16 rounding of each softmax weight shared by the variants, the
exponential's error, fp32 scores and fp32 accumulation; see mse_bound.py):
|mse_gpu - mse_oracle| <= mean(2 |D| b + b^2), which is proportional to mse
itself where the band holds most of the mass.
"""
import numpy as np
import pytest
import torch

import oracle
from mse_bound import mse_error_bounds
from sparse_attention_video_profile_b200 import svg, synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-5)}


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs = float(np.max(np.abs(got - ref)))
    rel_l2 = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    ta, tr = TOL[dtype]
    assert max_abs <= ta and rel_l2 <= tr, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel_l2:.3e}"


def rand_qkv(B, H, L, d, dtype, seed, scale=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return tuple((torch.randn(B, H, L, d, generator=g, device=DEV) * scale).to(dtype) for _ in range(3))


def sync_ok(status=None):
    torch.cuda.synchronize()
    if status is not None:
        assert int(status.item()) == 0, f"device status {int(status.item())}"


# ---------------------------------------------------------------- permute

@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 64), (torch.bfloat16, 128), (torch.float32, 32)])
@pytest.mark.parametrize("N,F", [(5, 37), (13, 1350), (1, 9), (7, 1)])
def test_permute_unpermute_bit_exact(dtype, d, N, F):
    B, H = 2, 3
    L = N * F
    x, _, _ = rand_qkv(B, H, L, d, dtype, 1)
    label = torch.tensor([[1, 0, 1], [0, 1, 1]], dtype=torch.int8, device=DEV)
    sentinel = torch.full_like(x, 7.0)
    xp = svg.svg_permute(x, N, F, label, out=sentinel.clone())
    back = svg.svg_unpermute(xp, N, F, label, out=sentinel.clone())
    torch.cuda.synchronize()
    xn, xpn, bn = f64(x), f64(xp), f64(back)
    ref = oracle.permute(xn, N, F)
    for b in range(B):
        for h in range(H):
            if label[b, h] == 1:
                np.testing.assert_array_equal(xpn[b, h], ref[b, h])
                np.testing.assert_array_equal(bn[b, h], xn[b, h])
            else:  # untouched
                assert np.all(xpn[b, h] == 7.0) and np.all(bn[b, h] == 7.0)
    # label = NULL: every head; the three-tensor launch gives the same bytes
    allp = svg.svg_permute(x, N, F, None)
    qp, kp, vp = svg.svg_permute_qkv(x, x, x, N, F, None)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(f64(allp), ref)
    for t in (qp, kp, vp):
        assert torch.equal(t, allp)


# ---------------------------------------------------------------- attention kernel

BAND_CASES = [  # (N, F, G, a)
    (3, 100, 100, 1),   # spatial-like, ragged L = 300 (one full + one partial CTA)
    (3, 100, 3, 5),     # temporal-like small groups
    (4, 64, 64, 1),     # the tiny shape
    (8, 256, 256, 2),   # the small shape, several key tiles
    (8, 256, 8, 16),
    (5, 61, 1, 1),      # diagonal only
    (5, 61, 7, 4),
    (2, 40, 80, 1),     # L = 80 < one tile
    (6, 300, 6, 1000),  # band wider than the sequence -> dense
]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("case", BAND_CASES, ids=lambda c: "N{}F{}G{}a{}".format(*c))
def test_banded_attention_bf16(d, case):
    N, F, G, a = case
    L = N * F
    q, k, v = rand_qkv(1, 2, L, d, torch.bfloat16, 2)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_banded_attn(q, k, v, N, F, G, a, status=status)
    sync_ok(status)
    qn, kn, vn = f64(q), f64(k), f64(v)
    mask = oracle.banded_mask(L, min(G, L), a)
    for h in range(2):
        ref = oracle.attention(qn[0, h], kn[0, h], vn[0, h], mask)
        assert_close(f64(o)[0, h], ref, torch.bfloat16, f"head {h}")


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("case", BAND_CASES[:6], ids=lambda c: "N{}F{}G{}a{}".format(*c))
def test_banded_attention_fp32(d, case):
    N, F, G, a = case
    L = N * F
    q, k, v = rand_qkv(1, 2, L, d, torch.float32, 3)
    o = svg.svg_banded_attn(q, k, v, N, F, G, a)
    sync_ok()
    mask = oracle.banded_mask(L, min(G, L), a)
    for h in range(2):
        ref = oracle.attention(f64(q)[0, h], f64(k)[0, h], f64(v)[0, h], mask)
        assert_close(f64(o)[0, h], ref, torch.float32, f"head {h}")


def test_diagonal_band_copies_values_exactly():
    """G = 1, a = 1 keeps only the self pair: softmax weight exactly 1, so the
    output is V itself, bit for bit."""
    q, k, v = rand_qkv(2, 3, 777, 128, torch.bfloat16, 4)
    o = svg.svg_banded_attn(q, k, v, 7, 111, 1, 1)
    sync_ok()
    assert torch.equal(o, v)


@pytest.mark.parametrize("d", [64, 128])
def test_masked_keys_weigh_exactly_zero(d):
    """G = 1, a = 1 keeps only the self pair; every other key of a tile is
    masked.  Odd rows of V hold 1e36: a masked key given any weight above 0
    (2^-125 would do: 1e36 * 2^-125 = 0.02 per key) would move the even rows'
    outputs, which must still equal V bit for bit.  Both exponential paths
    (MUFU and the FMA-pipe cubic) see masked keys."""
    q, k, v = rand_qkv(1, 2, 6 * 100, d, torch.bfloat16, 31)
    v[:, :, 1::2] = (torch.sign(v[:, :, 1::2]) * 1e36).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_banded_attn(q, k, v, 6, 100, 1, 1, status=status)
    sync_ok(status)
    assert torch.equal(o, v)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 64), (torch.bfloat16, 128), (torch.float32, 64)])
def test_dense_attention(dtype, d):
    N, F = 4, 77
    q, k, v = rand_qkv(1, 2, N * F, d, dtype, 5)
    o = svg.svg_dense_attn(q, k, v, N, F)
    sync_ok()
    ref = oracle.dense_attention(f64(q), f64(k), f64(v))
    assert_close(f64(o), ref, dtype, "dense")


def test_large_logits_stay_finite():
    """Scores spanning hundreds of units exercise the lazy-rescale path (Q and
    K scaled up; V keeps unit scale so the bf16 output grid stays fine)."""
    q, k, _ = rand_qkv(1, 2, 1024, 64, torch.bfloat16, 6, scale=4.0)
    _, _, v = rand_qkv(1, 2, 1024, 64, torch.bfloat16, 6)
    o = svg.svg_banded_attn(q, k, v, 4, 256, 256, 2)
    sync_ok()
    mask = oracle.banded_mask(1024, 256, 2)
    for h in range(2):
        ref = oracle.attention(f64(q)[0, h], f64(k)[0, h], f64(v)[0, h], mask)
        assert_close(f64(o)[0, h], ref, torch.bfloat16, f"head {h}")


# ---------------------------------------------------------------- labelled heads

@pytest.mark.parametrize("d", [64, 128])
def test_block_sparse_attn_with_labels(d):
    N, F, a1, a2 = 6, 90, 2, 7
    L = N * F
    q, k, v = rand_qkv(2, 2, L, d, torch.bfloat16, 7)
    label = torch.tensor([[0, 1], [1, 0]], dtype=torch.int8, device=DEV)
    qp, kp, vp = svg.svg_permute_qkv(q, k, v, N, F, label)
    o, op = svg.svg_block_sparse_attn(q, k, v, qp, kp, vp, label, N, F, a1, a2)
    out = svg.svg_unpermute(op, N, F, label, out=o)
    sync_ok()
    ref = oracle.sparse_attention(f64(q), f64(k), f64(v), label.cpu().numpy(), N, F, a1, a2)
    assert_close(f64(out), ref, torch.bfloat16, "block-sparse")


# ---------------------------------------------------------------- profiling

def profile_bounds(q, k, v, N, F, a1, a2, rows, fp32=False):
    """[B, H, 2] bounds on |mse_gpu - mse_oracle| (spatial, temporal) from the
    kernels' rounding, for fp64 inputs q, k, v [B, H, L, d]."""
    masks = [oracle.spatial_mask(N, F, min(a1, N), rows=rows), oracle.temporal_mask(N, F, min(a2, F), rows=rows)]
    B, H = q.shape[:2]
    out = np.zeros((B, H, 2))
    for b in range(B):
        for h in range(H):
            out[b, h] = mse_error_bounds(q[b, h], k[b, h], v[b, h], rows, masks, fp32_weights=fp32)[0]
    return out


def check_profile(mse, label, ref_mse, ref_label, bound):
    """MSEs within the rounding bound of the oracle's, head by head; labels
    equal wherever the oracle's gap exceeds 1e-3 relative (and wherever it
    exceeds the two bounds, which no rounding could cross)."""
    mse = mse.cpu().numpy().astype(np.float64)
    label = label.cpu().numpy()
    assert np.all(np.isfinite(mse)) and np.all(mse >= 0)
    err = np.abs(mse - ref_mse)
    worst = np.unravel_index(np.argmax(err / np.maximum(bound, 1e-300)), err.shape)
    assert np.all(err <= bound), f"mse {mse[worst]:.6e} vs oracle {ref_mse[worst]:.6e}, bound {bound[worst]:.3e}"
    gap_abs = np.abs(ref_mse[..., 0] - ref_mse[..., 1])
    decided = (gap_abs / np.maximum(ref_mse.max(-1), 1e-300) > 1e-3) | (gap_abs > bound.sum(-1))
    np.testing.assert_array_equal(label[decided], ref_label[decided])
    assert np.all(np.isin(label, [0, 1]))


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_profile_synthetic(name):
    wl = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(wl, seed=0, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, 0)
    rows = torch.from_numpy(rows_np).to(DEV)
    mse, label = svg.svg_profile_heads(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows)
    sync_ok()
    qn, kn, vn = f64(q), f64(k), f64(v)
    ref_mse, ref_label = oracle.profile_heads(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np)
    bound = profile_bounds(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np, fp32=q.dtype == torch.float32)
    check_profile(mse, label, ref_mse, ref_label, bound)
    np.testing.assert_array_equal(label.cpu().numpy(), synth.head_kinds(wl, 0))
    if name == "small":  # spatial heads with a small spatial MSE are covered
        assert ref_mse[..., 0].min() < 1e-4


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 64), (torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("S", [1, 17, 64, 128])
def test_profile_random(dtype, d, S):
    N, F, a1, a2 = 5, 133, 2, 11
    L = N * F
    q, k, v = rand_qkv(1, 3, L, d, dtype, 8 + S)
    rows_np = np.sort(np.random.default_rng(S).choice(L, S, replace=False)).astype(np.int32)
    rows = torch.from_numpy(rows_np).to(DEV)
    mse, label = svg.svg_profile_heads(q, k, v, N, F, a1, a2, rows)
    sync_ok()
    qn, kn, vn = f64(q), f64(k), f64(v)
    ref_mse, ref_label = oracle.profile_heads(qn, kn, vn, N, F, a1, a2, rows_np)
    check_profile(mse, label, ref_mse, ref_label,
                  profile_bounds(qn, kn, vn, N, F, a1, a2, rows_np, fp32=dtype == torch.float32))


def test_profile_special_cases_and_determinism():
    N, F = 4, 200
    q, k, v = rand_qkv(1, 2, N * F, 64, torch.bfloat16, 9)
    rows = torch.tensor([0, 5, 199, 200, 401, 799], dtype=torch.int32, device=DEV)
    mse, label = svg.svg_profile_heads(q, k, v, N, F, N, 3, rows)  # spatial band = all keys
    sync_ok()
    assert torch.all(mse[..., 0] == 0) and torch.all(mse[..., 1] > 0) and torch.all(label == 0)
    mse, label = svg.svg_profile_heads(q, k, v, N, F, 1, F, rows)  # temporal band = all keys
    sync_ok()
    assert torch.all(mse[..., 1] == 0) and torch.all(mse[..., 0] > 0) and torch.all(label == 1)
    a = svg.svg_profile_heads(q, k, v, N, F, 2, 5, rows)[0].clone()
    b = svg.svg_profile_heads(q, k, v, N, F, 2, 5, rows)[0].clone()
    sync_ok()
    assert torch.equal(a, b)


# ---------------------------------------------------------------- whole call

@pytest.mark.parametrize("name", ["tiny", "small"])
def test_sparse_3d_attn_end_to_end(name):
    wl = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(wl, seed=1, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, 1)
    rows = torch.from_numpy(rows_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, mse, label = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows, status=status)
    sync_ok(status)
    qn, kn, vn = f64(q), f64(k), f64(v)
    ref_mse, ref_label = oracle.profile_heads(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np)
    check_profile(mse, label, ref_mse, ref_label,
                  profile_bounds(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np, fp32=q.dtype == torch.float32))
    ref = oracle.sparse_attention(qn, kn, vn, label.cpu().numpy(), wl.N, wl.F, wl.a1, wl.a2)
    assert_close(f64(o), ref, q.dtype, name)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_sparse_3d_attn_literal_embedding_scale(name):
    """The whole call on the literal reading of the synthetic heads
    (embeddings N(0, 1) / sqrt(d), where the labels invert): profiling within
    the bound, labels as the oracle's, output within the bar."""
    wl = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(wl, seed=0, device=DEV, emb_std=wl.d ** -0.5)
    rows_np = synth.sample_rows(wl.L, wl.S, 0)
    rows = torch.from_numpy(rows_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, mse, label = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows, status=status)
    sync_ok(status)
    qn, kn, vn = f64(q), f64(k), f64(v)
    ref_mse, ref_label = oracle.profile_heads(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np)
    check_profile(mse, label, ref_mse, ref_label,
                  profile_bounds(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np, fp32=q.dtype == torch.float32))
    ref = oracle.sparse_attention(qn, kn, vn, label.cpu().numpy(), wl.N, wl.F, wl.a1, wl.a2)
    assert_close(f64(o), ref, q.dtype, name + " (literal embedding scale)")


def test_full_bands_equal_dense():
    wl = synth.WORKLOADS["small"]
    q, k, v = synth.make_qkv(wl, seed=2, device=DEV)
    rows = torch.from_numpy(synth.sample_rows(wl.L, wl.S, 2)).to(DEV)
    dense = svg.svg_dense_attn(q, k, v, wl.N, wl.F)
    ref = oracle.dense_attention(f64(q), f64(k), f64(v))
    for a1, a2 in ((wl.N, wl.a2), (wl.a1, wl.F), (wl.N, wl.F)):
        o, _, label = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, a1, a2, rows)
        sync_ok()
        assert_close(f64(o), ref, q.dtype, f"a1={a1} a2={a2}")
        full = (label.cpu().numpy() == 0) if a1 == wl.N else (label.cpu().numpy() == 1)
        if a1 == wl.N and a2 == wl.F:
            full[:] = True
        # heads whose band covers every key run the same tiles as dense: same bits
        dn, on = dense.cpu(), o.cpu()
        for b, h in zip(*np.nonzero(full)):
            if (label[b, h] == 0 and a1 == wl.N):
                assert torch.equal(on[b, h], dn[b, h])
    assert_close(f64(dense), ref, q.dtype, "dense")


# ---------------------------------------------------------------- video-model shapes

def sampled_rows(wl, n_extra=40, seed=0):
    """Rows at frame, tile and sequence boundaries plus random ones."""
    L, F, N = wl.L, wl.F, wl.N
    rows = {0, 1, L - 1, L - 2, F - 1, F, 127, 128, 255, 256, (L // 256) * 256, (L // 256) * 256 - 1}
    rows |= {i * F + j for i in (0, N // 2, N - 1) for j in (0, F - 1)}
    rows |= set(np.random.default_rng(seed).choice(L, n_extra, replace=False).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < L))


@pytest.mark.parametrize("name", ["cogvideox", "hunyuan"])
def test_video_shape_sampled(name):
    wl = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(wl, seed=0, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, 0)
    rows = torch.from_numpy(rows_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, mse, label = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows, status=status)
    sync_ok(status)
    label_np = label.cpu().numpy()
    mse_np = mse.cpu().numpy()
    check_rows = sampled_rows(wl)
    heads = range(wl.H) if name == "cogvideox" else range(0, wl.H, 3)
    for h in range(wl.H):
        qn, kn, vn = (f64(t[:, h:h + 1]) for t in (q, k, v))
        ref_mse, ref_label = oracle.profile_heads(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np)
        check_profile(torch.from_numpy(mse_np[:, h:h + 1]), torch.from_numpy(label_np[:, h:h + 1]),
                      ref_mse, ref_label, profile_bounds(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np))
        if h in heads:
            ref = oracle.sparse_attention(qn, kn, vn, label_np[:, h:h + 1], wl.N, wl.F, wl.a1, wl.a2,
                                          rows=check_rows)
            got = f64(o[:, h:h + 1, torch.from_numpy(check_rows).to(DEV)])
            assert_close(got, ref, q.dtype, f"{name} head {h}")
    assert set(np.unique(label_np)) <= {0, 1}


@pytest.mark.parametrize("density", [0.05, 0.5])
def test_density_sweep_extremes_sampled(density):
    """HunyuanVideo shape at the ends of the 5-50 % sweep: at 5 % the whole
    call keeps the separate layout, at 50 % the fused one with a wide band
    (a2 = 1055).  One spatial and one temporal head: profiling against the
    oracle, and sampled output rows against the oracle."""
    a1, a2 = synth.HUNYUAN_SWEEP[density]
    wl = synth.WORKLOADS["hunyuan"].with_bands(a1, a2)
    q, k, v = synth.make_qkv(wl, seed=3, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, 3)
    rows = torch.from_numpy(rows_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, mse, label = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows, status=status)
    sync_ok(status)
    label_np = label.cpu().numpy()
    mse_np = mse.cpu().numpy()
    heads = [int(np.flatnonzero(label_np[0] == kind)[0]) for kind in (0, 1) if (label_np[0] == kind).any()]
    check_rows = sampled_rows(wl, n_extra=16)
    for h in heads:
        qn, kn, vn = (f64(t[:, h:h + 1]) for t in (q, k, v))
        ref_mse, ref_label = oracle.profile_heads(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np)
        check_profile(torch.from_numpy(mse_np[:, h:h + 1]), torch.from_numpy(label_np[:, h:h + 1]),
                      ref_mse, ref_label, profile_bounds(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np))
        ref = oracle.sparse_attention(qn, kn, vn, label_np[:, h:h + 1], wl.N, wl.F, wl.a1, wl.a2, rows=check_rows)
        got = f64(o[:, h:h + 1, torch.from_numpy(check_rows).to(DEV)])
        assert_close(got, ref, q.dtype, f"density {density} head {h}")


# ---------------------------------------------------------------- failure detection

def _underflow_inputs(N, F, d):
    """Q and K such that a sampled row of frame 0 has every spatial in-band
    logit (its own frame, a1 = 1) more than 126 / (scale log2 e) below the
    largest logit of the same key chunk (a key of frame 1; with F = 64 both
    frames lie in the first 128-key tile): the profiling kernel cannot weigh
    the in-band keys against that shared reference and reports SVG_DEV_RANGE."""
    L = N * F
    q = torch.full((1, 2, L, d), 12.0)
    k = torch.zeros(1, 2, L, d)
    k[:, :, F:2 * F] = 12.0  # scores 144 d / sqrt(d) = 1152 at d = 64, far above the 698 threshold
    v = torch.randn(1, 2, L, d, generator=torch.Generator().manual_seed(5))
    return tuple(t.to(torch.bfloat16).to(DEV) for t in (q, k, v))


def test_profiling_failure_reaches_status_and_runs_spatial_in_both_layouts():
    """A profiling failure (in-band weights that underflow) labels every head
    -1 with NaN MSEs; the whole call ORs SVG_DEV_RANGE into the caller's
    status word and runs every head with the spatial band, in the fused and
    in the separate layout (and from host buffers), so both give the oracle's
    spatial attention."""
    N, F, d, a1 = 5, 64, 64, 1  # a shape whose layout choice depends on a2
    L = N * F
    q, k, v = _underflow_inputs(N, F, d)
    rows_np = np.array([3, 70, 130, 200], dtype=np.int32)
    rows = torch.from_numpy(rows_np).to(DEV)
    ref = oracle.sparse_attention(f64(q), f64(k), f64(v), np.zeros((1, 2), np.int8), N, F, a1, 1)
    layouts = {}
    for a2 in range(1, F + 1):  # one band of each layout choice
        fused = svg.svg_sparse_3d_attn_plan(svg.make_shape(q, N, F), a2)[2]
        layouts.setdefault(fused, a2)
    assert set(layouts) == {0, 1}, layouts
    for fused, a2 in sorted(layouts.items()):
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        o, mse, label = svg.svg_sparse_3d_attn(q, k, v, N, F, a1, a2, rows, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == svg.SVG_DEV_RANGE, (fused, int(status.item()))
        assert torch.all(label == -1) and torch.all(torch.isnan(mse))
        assert_close(f64(o), ref, torch.bfloat16, f"fused={fused}")
        status.zero_()
        o_h, mse_h, lab_h = svg.svg_sparse_3d_attn_host(q.cpu().pin_memory(), k.cpu().pin_memory(),
                                                        v.cpu().pin_memory(), N, F, a1, a2, torch.from_numpy(rows_np),
                                                        heads_per_chunk=1, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == svg.SVG_DEV_RANGE
        assert torch.equal(o_h, o.cpu()) and torch.all(lab_h == -1)
    # the stand-alone profiling call keeps the failure in its own workspace
    mse, label = svg.svg_profile_heads(q, k, v, N, F, a1, 8, rows)
    torch.cuda.synchronize()
    assert torch.all(label == -1) and torch.all(torch.isnan(mse))
    # and a later call on sound inputs is not affected by it
    q2, k2, v2 = rand_qkv(1, 2, L, d, torch.bfloat16, 6)
    mse2, label2 = svg.svg_profile_heads(q2, k2, v2, N, F, a1, 8, rows)
    torch.cuda.synchronize()
    assert torch.all(label2 >= 0) and torch.all(torch.isfinite(mse2))


def test_bounded_waits_report_timeout_and_context_stays_usable():
    """The attention kernel with its loads withheld: every wait gives up after
    50 ms, the status word reports the timeout, and the next call is normal."""
    q, k, v = rand_qkv(1, 2, 4 * 700, 128, torch.bfloat16, 21)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    svg.svg_selftest_wait_bound(q, k, v, 4, 700, status, wait_ns=50_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) & svg.SVG_DEV_TIMEOUT
    status.zero_()
    o = svg.svg_dense_attn(q, k, v, 4, 700, status=status)
    sync_ok(status)
    ref = oracle.dense_attention(f64(q), f64(k), f64(v))
    assert_close(f64(o), ref, torch.bfloat16, "after timeout")


# ---------------------------------------------------------------- mixed sparse patterns

@pytest.mark.parametrize("d", [64, 128])
def test_mixed_patterns_small(d):
    N, F = 6, 90
    L = N * F
    modes_np = np.array([[0, 1, 2, 3, 4, 2, 3, 4, 0, 2]], dtype=np.int8)
    q, k, v = rand_qkv(1, 10, L, d, torch.bfloat16, 23)
    mode = torch.from_numpy(modes_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_mixed_3d_attn(q, k, v, mode, N, F, F, 7, 100, status=status)
    sync_ok(status)
    ref = oracle.mixed_attention(f64(q), f64(k), f64(v), modes_np, N, F, F, 7, 100)
    assert_close(f64(o), ref, torch.bfloat16, "mixed")
    assert torch.all(o[0, 1] == 0)


def test_mixed_workload_sampled():
    wl = synth.WORKLOADS["mixed"]
    prm = synth.MIXED_PARAMS
    q, k, v = synth.make_qkv(wl, seed=0, device=DEV)
    modes_np = synth.head_modes(wl.B, wl.H, 0)
    mode = torch.from_numpy(modes_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_mixed_3d_attn(q, k, v, mode, wl.N, wl.F, prm["window"], prm["md_half"], prm["stripe"],
                              status=status)
    sync_ok(status)
    rows = sampled_rows(wl, n_extra=24)
    idx = torch.from_numpy(rows).to(DEV)
    for h in range(wl.H):
        qn, kn, vn = (f64(t[:, h:h + 1]) for t in (q, k, v))
        ref = oracle.mixed_attention(qn, kn, vn, modes_np[:, h:h + 1], wl.N, wl.F, prm["window"],
                                     prm["md_half"], prm["stripe"], rows=rows)
        assert_close(f64(o[:, h:h + 1, idx]), ref, q.dtype, f"mixed head {h} mode {modes_np[0, h]}")


# ---------------------------------------------------------------- head-sharded call

@pytest.mark.parametrize("world", [2, 3])
def test_head_shards_assemble_the_whole_call(world):
    """Each rank's block of heads (svg_sparse_3d_attn_shard), run here one
    rank after another on one GPU into the same full-size tensors, gives the
    single whole call: the same outputs bit for bit and the same labels (per
    head the attention does not depend on the other heads); the MSEs within
    the rounding bound (the profiling's key split depends on the head count)."""
    wl = synth.WORKLOADS["small"]
    q, k, v = synth.make_qkv(wl, seed=8, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, 8)
    rows = torch.from_numpy(rows_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o_ref, mse_ref, lab_ref = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows, status=status)
    o = torch.full_like(q, float("nan"))
    mse = torch.full_like(mse_ref, float("nan"))
    lab = torch.full_like(lab_ref, -7)
    for r in range(world):
        svg.svg_sparse_3d_attn_shard(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows, r, world, o=o, mse=mse, label=lab,
                                     status=status)
    sync_ok(status)
    assert torch.equal(lab, lab_ref)
    assert torch.equal(o, o_ref)
    qn, kn, vn = f64(q), f64(k), f64(v)
    bound = profile_bounds(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np)
    assert np.all(np.abs(mse.cpu().double().numpy() - mse_ref.cpu().double().numpy()) <= 2 * bound)


# ---------------------------------------------------------------- host-buffer call

@pytest.mark.parametrize("hc", [1, 3, 8])
def test_host_pipeline_bit_identical(hc):
    wl = synth.WORKLOADS["small"]
    q, k, v = synth.make_qkv(wl, seed=5, device=DEV)
    rows = torch.from_numpy(synth.sample_rows(wl.L, wl.S, 5))
    o_dev, mse_dev, lab_dev = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows.to(DEV))
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o_h, mse_h, lab_h = svg.svg_sparse_3d_attn_host(qh, kh, vh, wl.N, wl.F, wl.a1, wl.a2, rows, heads_per_chunk=hc,
                                                    status=status)
    sync_ok(status)
    assert torch.equal(o_h, o_dev.cpu())
    assert torch.equal(mse_h, mse_dev.cpu())
    assert torch.equal(lab_h, lab_dev.cpu())


# ---------------------------------------------------------------- offline mode search

def mode_bounds(q, k, v, N, F, rows, window, md_half, stripe):
    """[B, H, 4] bounds on |mse_gpu - mse_oracle| of the four sparse modes
    (skip, diagonal, multi-diagonal, stripe), from the kernels' rounding."""
    masks = [oracle.mode_mask(m, N, F, window, md_half, stripe, rows=rows) for m in oracle.SEARCH_MODES]
    B, H = q.shape[:2]
    out = np.zeros((B, H, 4))
    for b in range(B):
        for h in range(H):
            out[b, h] = mse_error_bounds(q[b, h], k[b, h], v[b, h], rows, masks)[0]
    return out


def check_mode_search(loss, mode, ref_loss, ref_mode, sp, lam, eps, bound):
    """The MSE part of each loss (L_i - lambda (1 - S_i)) within the rounding
    bound of the oracle's, plus the fp32 rounding of the loss itself; modes
    equal wherever the oracle's decision has a margin larger than those
    bounds."""
    loss = loss.cpu().numpy().astype(np.float64)
    mode = mode.cpu().numpy()
    assert np.all(np.isfinite(loss))
    pen = lam * (1.0 - np.asarray(sp))
    err = bound + 4 * 2.0 ** -24 * (np.abs(ref_loss) + 1.0)  # fp32 loss and penalty
    got_mse, ref_mse = loss - pen, ref_loss - pen
    assert np.all(np.abs(got_mse - ref_mse) <= err), float(np.max(np.abs(got_mse - ref_mse) / err))
    order = np.argsort(ref_loss, -1)
    srt = np.take_along_axis(ref_loss, order, -1)
    e_srt = np.take_along_axis(err, order, -1)
    decided = (srt[..., 1] - srt[..., 0] > e_srt[..., 0] + e_srt[..., 1]) & (np.abs(srt[..., 0] - eps) > e_srt[..., 0])
    np.testing.assert_array_equal(mode[decided], ref_mode[decided])
    assert np.all(np.isin(mode, [0, 1, 2, 3, 4]))
    return decided


def test_mode_search_structured():
    """Attention one-hot on the key one mode keeps: that mode must win."""
    N, F, d = 2, 32, 64
    L = N * F
    targets = [lambda x: x, lambda x: ((x // F + 1) % N) * F + x % F, lambda x: 0]
    q = torch.zeros(1, 3, L, d)
    k = torch.eye(L, d).expand(1, 3, L, d).contiguous()
    for h, t in enumerate(targets):
        for x in range(L):
            q[0, h, x, t(x)] = 40.0 * 8.0  # logit 40 after the 1/sqrt(d) scale
    v = torch.randn(1, 3, L, d, generator=torch.Generator().manual_seed(3))
    q, k, v = (t.to(torch.bfloat16).to(DEV) for t in (q, k, v))
    rows_np = np.arange(0, L, 3, dtype=np.int32)
    rows = torch.from_numpy(rows_np).to(DEV)
    loss, mode = svg.svg_mode_search(q, k, v, N, F, rows, 0, 0, 1)
    sync_ok()
    ref_loss, ref_mode = oracle.mode_search(f64(q), f64(k), f64(v), N, F, rows_np, 0, 0, 1)
    sp = [oracle.mode_sparsity(m, N, F, 0, 0, 1) for m in oracle.SEARCH_MODES]
    check_mode_search(loss, mode, ref_loss, ref_mode, sp, 0.5, 1.0, mode_bounds(f64(q), f64(k), f64(v), N, F, rows_np, 0, 0, 1))
    np.testing.assert_array_equal(mode.cpu().numpy()[0], [svg.MODE_DIAGONAL, svg.MODE_MULTIDIAG, svg.MODE_STRIPE])
    _, mode = svg.svg_mode_search(q, k, v, N, F, rows, 0, 0, 1, epsilon=0.005)  # every L_i >= lam / L = 0.0078
    sync_ok()
    assert torch.all(mode == svg.MODE_FULL)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("S", [17, 128])
def test_mode_search_random(d, S):
    N, F, W, h, P = 6, 90, 90, 7, 100
    L = N * F
    q, k, v = rand_qkv(2, 3, L, d, torch.bfloat16, 40 + S)
    rows_np = np.sort(np.random.default_rng(S).choice(L, S, replace=False)).astype(np.int32)
    rows = torch.from_numpy(rows_np).to(DEV)
    bound = mode_bounds(f64(q), f64(k), f64(v), N, F, rows_np, W, h, P)
    for lam, eps in [(0.5, 1.0), (0.05, 0.3)]:
        loss, mode = svg.svg_mode_search(q, k, v, N, F, rows, W, h, P, lam=lam, epsilon=eps)
        sync_ok()
        ref_loss, ref_mode = oracle.mode_search(f64(q), f64(k), f64(v), N, F, rows_np, W, h, P, lam=lam, eps=eps)
        sp = [oracle.mode_sparsity(m, N, F, W, h, P) for m in oracle.SEARCH_MODES]
        check_mode_search(loss, mode, ref_loss, ref_mode, sp, lam, eps, bound)


def test_mode_search_mixed_workload():
    wl = synth.WORKLOADS["mixed"]
    prm = synth.MIXED_PARAMS
    q, k, v = synth.make_qkv(wl, seed=0, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, 0)
    rows = torch.from_numpy(rows_np).to(DEV)
    args = (wl.N, wl.F, prm["window"], prm["md_half"], prm["stripe"])
    loss, mode = svg.svg_mode_search(q, k, v, wl.N, wl.F, rows, *args[2:])
    loss2, mode2 = svg.svg_mode_search(q, k, v, wl.N, wl.F, rows, *args[2:])
    sync_ok()
    assert torch.equal(loss, loss2) and torch.equal(mode, mode2)  # deterministic
    sp = [oracle.mode_sparsity(m, *args) for m in oracle.SEARCH_MODES]
    ref_loss, ref_mode = oracle.mode_search(f64(q), f64(k), f64(v), wl.N, wl.F, rows_np, *args[2:], sparsity=sp)
    bound = mode_bounds(f64(q), f64(k), f64(v), wl.N, wl.F, rows_np, *args[2:])
    decided = check_mode_search(loss, mode, ref_loss, ref_mode, sp, 0.5, 1.0, bound)
    assert decided.mean() > 0.5


# ---------------------------------------------------------------- fused layout transformation

@pytest.mark.parametrize("N,F,d", [(6, 90, 128), (5, 133, 64), (33, 17, 128), (1, 300, 128), (7, 1, 64),
                                   (3, 29, 128), (13, 45, 64), (21, 20, 128), (130, 3, 64)])
def test_fused_block_sparse(N, F, d):
    """Frame-group boxes (s frames x 128/s positions per tile) from the
    frame-major tensors and the frame-major output scatter: against the
    oracle, on shapes with 1..8 frame groups, ragged position tails and
    frames above 128."""
    L = N * F
    H = 4
    q, k, v = rand_qkv(2, H, L, d, torch.bfloat16, 50 + N + F)
    label = torch.tensor([[1, 0, 1, 1], [0, 1, 0, 1]], dtype=torch.int8, device=DEV)
    a1, a2 = min(2, N), max(1, min(F, 7))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_block_sparse_attn_fused(q, k, v, label, N, F, a1, a2, status=status)
    sync_ok(status)
    ref = oracle.sparse_attention(f64(q), f64(k), f64(v), label.cpu().numpy(), N, F, a1, a2)
    assert_close(f64(o), ref, torch.bfloat16, "fused")


def test_fused_matches_separate_layout_video_shape():
    """HunyuanVideo shape: the whole call (fused layout) against profile ->
    permute -> attention -> unpermute; same labels and MSEs bit for bit (same
    profiling), outputs within twice the bf16 tolerance of each other, and
    sampled rows against the oracle."""
    wl = synth.WORKLOADS["hunyuan"]
    q, k, v = synth.make_qkv(wl, seed=2, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, 2)
    rows = torch.from_numpy(rows_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, mse, lab = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows, status=status)
    mse2, lab2 = svg.svg_profile_heads(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows)
    qp, kp, vp = svg.svg_permute_qkv(q, k, v, wl.N, wl.F, lab2)
    o2, op = svg.svg_block_sparse_attn(q, k, v, qp, kp, vp, lab2, wl.N, wl.F, wl.a1, wl.a2, status=status)
    o2 = svg.svg_unpermute(op, wl.N, wl.F, lab2, out=o2)
    sync_ok(status)
    del qp, kp, vp, op
    assert torch.equal(lab, lab2) and torch.equal(mse, mse2)
    assert int(lab.sum()) > 0  # the token-major path is exercised
    # each path is within (2e-2 max-abs, 1e-2 rel L2) of the exact result, so
    # by the triangle inequality they are within twice that of each other
    diff = (o.float() - o2.float())
    assert float(diff.abs().max()) <= 4e-2, float(diff.abs().max())
    assert float(diff.norm() / o2.float().norm()) <= 2e-2
    idx = torch.from_numpy(sampled_rows(wl, n_extra=16)).to(DEV)
    for h in range(wl.H):
        if int(lab[0, h]) == 0:
            continue
        qn, kn, vn = (f64(t[:, h:h + 1]) for t in (q, k, v))
        ref = oracle.sparse_attention(qn, kn, vn, lab[:, h:h + 1].cpu().numpy(), wl.N, wl.F, wl.a1, wl.a2,
                                      rows=idx.cpu().numpy())
        assert_close(f64(o[:, h:h + 1, idx]), ref, q.dtype, f"fused head {h}")
        break


@pytest.mark.parametrize("name", ["small", "mixed"])
def test_fused_mixed(name):
    if name == "small":
        N, F, H, d = 6, 90, 10, 128
        q, k, v = rand_qkv(1, H, N * F, d, torch.bfloat16, 61)
        modes_np = np.array([[0, 1, 2, 3, 4, 3, 3, 4, 0, 2]], dtype=np.int8)
        win, mdh, stripe = F, 7, 100
        rows = None
    else:
        wl = synth.WORKLOADS["mixed"]
        prm = synth.MIXED_PARAMS
        N, F = wl.N, wl.F
        q, k, v = synth.make_qkv(wl, seed=1, device=DEV)
        modes_np = synth.head_modes(wl.B, wl.H, 1)
        win, mdh, stripe = prm["window"], prm["md_half"], prm["stripe"]
        rows = sampled_rows(wl, n_extra=12)
    mode = torch.from_numpy(modes_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_mixed_attn_fused(q, k, v, mode, N, F, win, mdh, stripe, status=status)
    sync_ok(status)
    if rows is None:
        ref = oracle.mixed_attention(f64(q), f64(k), f64(v), modes_np, N, F, win, mdh, stripe)
        assert_close(f64(o), ref, torch.bfloat16, "fused mixed")
        return
    idx = torch.from_numpy(rows).to(DEV)
    for h in np.nonzero(modes_np[0] == 3)[0][:3]:
        qn, kn, vn = (f64(t[:, h:h + 1]) for t in (q, k, v))
        ref = oracle.mixed_attention(qn, kn, vn, modes_np[:, h:h + 1], N, F, win, mdh, stripe, rows=rows)
        assert_close(f64(o[:, h:h + 1, idx]), ref, q.dtype, f"fused mixed head {h}")


def test_fused_rejects_fp32():
    q, k, v = rand_qkv(1, 1, 64, 64, torch.float32, 3)
    label = torch.zeros(1, 1, dtype=torch.int8, device=DEV)
    with pytest.raises(svg.SvgError):
        svg.svg_block_sparse_attn_fused(q, k, v, label, 4, 16, 1, 1)


# ---------------------------------------------------------------- SVG2 semantic-aware attention

def _cluster_means(x, assign, C):
    mu = np.zeros((C, x.shape[1]))
    n = np.bincount(assign, minlength=C)
    np.add.at(mu, assign, x)
    mu[n > 0] /= n[n > 0, None]
    return mu, n


def _check_topp_valid(sel, mu_q, mu_k, n_k, p, scale, tol=2e-4):
    """The GPU's kept set for each query cluster against fp64 masses of the
    same clusters: mass >= p, minimal, and heaviest (each to `tol`, the fp32
    rounding of the GPU's masses and cumulative sum)."""
    logits = scale * mu_q @ mu_k.T
    w = np.where(n_k[None] > 0, n_k[None] * np.exp(logits - logits.max(1, keepdims=True)), 0.0)
    w = w / w.sum(1, keepdims=True)
    for c in range(sel.shape[0]):
        kept, left = np.nonzero(sel[c])[0], np.nonzero(~sel[c])[0]
        assert len(kept) > 0 and np.all(n_k[kept] > 0)
        mass = w[c, kept].sum()
        assert mass >= p - tol, (c, mass)
        assert mass - w[c, kept].min() < p + tol, (c, mass)
        if len(left):
            assert w[c, kept].min() >= w[c, left].max() - tol


def _semantic_inputs(B, H, N, F, d, Cq, Ck, seed, iters=3):
    q, k, v = rand_qkv(B, H, N * F, d, torch.bfloat16, seed)
    qn, kn = f64(q), f64(k)
    aq = np.stack([[oracle.kmeans(qn[b, h], Cq, iters)[0] for h in range(H)] for b in range(B)]).astype(np.int32)
    ak = np.stack([[oracle.kmeans(kn[b, h], Ck, iters)[0] for h in range(H)] for b in range(B)]).astype(np.int32)
    return q, k, v, aq, ak


@pytest.mark.parametrize("N,F,d,Cq,Ck,p", [(4, 300, 128, 8, 24, 0.9), (3, 211, 64, 5, 40, 0.6), (2, 700, 128, 16, 64, 0.95),
                                           (1, 100, 64, 3, 7, 0.5)])
def test_semantic_attention(N, F, d, Cq, Ck, p):
    B, H = 1, 2
    q, k, v, aq, ak = _semantic_inputs(B, H, N, F, d, Cq, Ck, 70 + F)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    aq_t, ak_t = (torch.from_numpy(a).to(DEV) for a in (aq, ak))
    o, sel = svg.svg_semantic_attn(q, k, v, N, F, aq_t, ak_t, Cq, Ck, p, status=status)
    o2, sel2 = svg.svg_semantic_attn(q, k, v, N, F, aq_t, ak_t, Cq, Ck, p, status=status)
    sync_ok(status)
    assert torch.equal(o, o2) and torch.equal(sel, sel2)  # deterministic
    bits = svg.selected_bits(sel, Ck)
    scale = 1.0 / np.sqrt(d)
    for h in range(H):
        qh, kh, vh = f64(q)[0, h], f64(k)[0, h], f64(v)[0, h]
        mu_q, _ = _cluster_means(qh, aq[0, h], Cq)
        mu_k, n_k = _cluster_means(kh, ak[0, h], Ck)
        _check_topp_valid(bits[0, h], mu_q, mu_k, n_k, p, scale)
        ref = oracle.svg2_attention_given(qh, kh, vh, aq[0, h], ak[0, h], bits[0, h])
        assert_close(f64(o[0, h]), ref, torch.bfloat16, f"semantic head {h}")


def test_semantic_attention_single_small_key_cluster():
    """Every query keeps one key cluster of three keys (its centroid score
    dominates the top-p mass); the other keys hold V = 1e36, so any weight
    above 0 on a key outside the kept cluster would show in the output."""
    N, F, d, Cq, Ck = 2, 128, 64, 1, 4
    L = N * F
    g = torch.Generator().manual_seed(12)
    q = torch.ones(1, 1, L, d) + 0.01 * torch.randn(1, 1, L, d, generator=g)
    k = 0.01 * torch.randn(1, 1, L, d, generator=g)
    v = torch.randn(1, 1, L, d, generator=g)
    kept = [5, 77, 200]
    k[0, 0, kept] = 8.0 + 0.5 * torch.randn(3, d, generator=g)
    others = np.setdiff1d(np.arange(L), kept)
    v[0, 0, others] = torch.sign(v[0, 0, others]) * 1e36
    ak = (np.arange(L) % 3 + 1).astype(np.int32)
    ak[kept] = 0
    aq = np.zeros(L, np.int32)
    q, k, v = (t.to(torch.bfloat16).to(DEV) for t in (q, k, v))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, sel = svg.svg_semantic_attn(q, k, v, N, F, torch.from_numpy(aq[None, None]).to(DEV),
                                   torch.from_numpy(ak[None, None]).to(DEV), Cq, Ck, 0.9, status=status)
    sync_ok(status)
    bits = svg.selected_bits(sel, Ck)
    np.testing.assert_array_equal(bits[0, 0, 0], [True, False, False, False])
    ref = oracle.svg2_attention_given(f64(q)[0, 0], f64(k)[0, 0], f64(v)[0, 0], aq, ak, bits[0, 0])
    assert_close(f64(o[0, 0]), ref, torch.bfloat16, "single kept cluster")


def test_semantic_attention_p1_is_dense_and_bad_ids_flagged():
    N, F, d, Cq, Ck = 3, 200, 128, 6, 20
    q, k, v, aq, ak = _semantic_inputs(1, 2, N, F, d, Cq, Ck, 81)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, sel = svg.svg_semantic_attn(q, k, v, N, F, torch.from_numpy(aq).to(DEV), torch.from_numpy(ak).to(DEV), Cq, Ck,
                                   1.0, status=status)
    sync_ok(status)
    bits = svg.selected_bits(sel, Ck)
    nonempty = np.stack([np.bincount(ak[0, h], minlength=Ck) > 0 for h in range(2)])
    np.testing.assert_array_equal(bits[0], np.repeat(nonempty[:, None, :], Cq, axis=1))
    assert_close(f64(o), oracle.dense_attention(f64(q), f64(k), f64(v)), torch.bfloat16, "p = 1")
    bad = aq.copy()
    bad[0, 1, 17] = Cq + 5
    status.zero_()
    svg.svg_semantic_attn(q, k, v, N, F, torch.from_numpy(bad).to(DEV), torch.from_numpy(ak).to(DEV), Cq, Ck, 0.9,
                          status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & svg.SVG_DEV_RANGE


def test_semantic_attention_video_shape_sampled():
    """HunyuanVideo shape, Cq = 128, Ck = 512, hashed cluster ids: sampled
    rows of two heads against the oracle under the GPU's selection."""
    wl = synth.WORKLOADS["hunyuan"]
    Cq, Ck, p = 128, 512, 0.9
    q, k, v = synth.make_qkv(wl, seed=3, device=DEV)
    x = np.arange(wl.L, dtype=np.int64)
    aq = np.stack([((x * 2654435761 + 97 * h) >> 7) % Cq for h in range(wl.H)]).astype(np.int32)[None]
    ak = np.stack([((x * 40503 + 31 * h) >> 5) % Ck for h in range(wl.H)]).astype(np.int32)[None]
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, sel = svg.svg_semantic_attn(q, k, v, wl.N, wl.F, torch.from_numpy(aq).to(DEV), torch.from_numpy(ak).to(DEV),
                                   Cq, Ck, p, status=status)
    sync_ok(status)
    bits = svg.selected_bits(sel, Ck)
    rows = sampled_rows(wl, n_extra=12)
    idx = torch.from_numpy(rows).to(DEV)
    for h in (0, 17):
        qh, kh, vh = f64(q)[0, h], f64(k)[0, h], f64(v)[0, h]
        ref = oracle.svg2_attention_given(qh, kh, vh, aq[0, h], ak[0, h], bits[0, h], rows=rows)
        assert_close(f64(o[0, h, idx]), ref, torch.bfloat16, f"semantic video head {h}")


# ---------------------------------------------------------------- k-means and the whole SVG2-style call

@pytest.mark.parametrize("d", [64, 128])
def test_kmeans_recovers_blobs(d):
    """Blobs ordered by row, so the start rows floor(c L / C) are one per
    blob: every round assigns each row to its blob exactly."""
    C, per, H = 12, 64, 2
    rng = np.random.default_rng(d)
    xs, labs = [], []
    for h in range(H):
        centers = rng.standard_normal((C, d)) * 4.0
        xs.append(np.concatenate([centers[c] + 0.05 * rng.standard_normal((per, d)) for c in range(C)]))
        labs.append(np.repeat(np.arange(C), per))
    x = torch.from_numpy(np.stack(xs)[None]).to(torch.bfloat16).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    assign, mu = svg.svg_kmeans(x, 1, C * per, C, 3, status=status)
    sync_ok(status)
    xn = f64(x)[0]
    for h in range(H):
        np.testing.assert_array_equal(assign.cpu().numpy()[0, h], labs[h])
        for c in range(C):
            np.testing.assert_allclose(mu.cpu().numpy()[0, h, c], xn[h][labs[h] == c].mean(0), rtol=0, atol=1e-5)


def _check_nearest(x, c, assign):
    """Every row's cluster is its nearest centroid of c, up to the fp32
    rounding of the GPU's score ||c||^2 - 2 x.c (a d-term fp32 norm and a
    d-term dot product accumulated in fp32, then one fp32 subtraction)."""
    d = x.shape[1]
    score = (c * c).sum(1)[None, :] - 2.0 * x @ c.T
    mag = (c * c).sum(1)[None, :] + 2.0 * np.abs(x) @ np.abs(c).T
    tol = (d + 4) * 2.0 ** -23 * mag
    rows = np.arange(x.shape[0])
    best = score.min(1)
    ok = score[rows, assign] <= best + tol[rows, assign] + tol[rows, score.argmin(1)]
    assert np.all(ok), int(np.flatnonzero(~ok)[0])


@pytest.mark.parametrize("d,C", [(128, 40), (64, 300), (128, 512)])
def test_kmeans_one_round_and_several(d, C):
    N, F, H = 3, 700, 2
    q, _, _ = rand_qkv(1, H, N * F, d, torch.bfloat16, 90 + C)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    a1, mu1 = svg.svg_kmeans(q, N, F, C, 1, status=status)
    a4, mu4 = svg.svg_kmeans(q, N, F, C, 4, status=status)
    a5, mu5 = svg.svg_kmeans(q, N, F, C, 5, status=status)
    a5b, mu5b = svg.svg_kmeans(q, N, F, C, 5, status=status)
    sync_ok(status)
    assert torch.equal(a5, a5b) and torch.equal(mu5, mu5b)  # deterministic
    L = N * F
    init = (np.arange(C) * L) // C
    for h in range(H):
        x = f64(q)[0, h]
        # one round: the nearest start row (bf16 start rows are exact), up to rounding of the scores
        d2 = ((x[:, None, :] - x[init][None, :, :]) ** 2).sum(-1)
        g = a1.cpu().numpy()[0, h]
        gap = d2[np.arange(L), g] - d2.min(1)
        assert np.all(gap <= 1e-3 * (1.0 + d2.min(1))), float(gap.max())
        ref_mu, n = _cluster_means(x, g, C)
        got = mu1.cpu().numpy()[0, h]
        np.testing.assert_allclose(got[n > 0], ref_mu[n > 0], rtol=0, atol=2e-5)
        np.testing.assert_array_equal(got[n == 0], x[init][n == 0])  # empty clusters keep their start row
        # five rounds, row by row: the fifth assignment puts every row at its
        # nearest centroid of the fourth round's update (the centroids a
        # four-round call returns), rounded to bf16 as the GPU multiplies
        # them, within the fp32 rounding of the scores; the returned
        # centroids are the fp64 means of that assignment (empty clusters keep
        # the fourth round's centroid)
        g5 = a5.cpu().numpy()[0, h]
        c4 = mu4.to(torch.bfloat16).double().cpu().numpy()[0, h]
        _check_nearest(x, c4, g5)
        ref_mu5, n5 = _cluster_means(x, g5, C)
        got5 = mu5.cpu().numpy()[0, h]
        np.testing.assert_allclose(got5[n5 > 0], ref_mu5[n5 > 0], rtol=0, atol=2e-5)
        np.testing.assert_array_equal(got5[n5 == 0], mu4.cpu().numpy()[0, h][n5 == 0])
        # and the objective is that of a Lloyd run: no worse than the start rows' one
        start_obj = oracle.kmeans_objective(x, x[init], a1.cpu().numpy()[0, h])
        assert oracle.kmeans_objective(x, ref_mu5, g5) <= start_obj * (1 + 1e-6)


def test_semantic_3d_attn_whole_call():
    N, F, d, Cq, Ck, p = 4, 300, 128, 10, 40, 0.9
    q, k, v = rand_qkv(1, 2, N * F, d, torch.bfloat16, 95)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, aq, ak, sel = svg.svg_semantic_3d_attn(q, k, v, N, F, Cq, Ck, 4, p, status=status)
    sync_ok(status)
    aq, ak = aq.cpu().numpy(), ak.cpu().numpy()
    bits = svg.selected_bits(sel, Ck)
    for h in range(2):
        qh, kh, vh = f64(q)[0, h], f64(k)[0, h], f64(v)[0, h]
        mu_q, _ = _cluster_means(qh, aq[0, h], Cq)
        mu_k, n_k = _cluster_means(kh, ak[0, h], Ck)
        _check_topp_valid(bits[0, h], mu_q, mu_k, n_k, p, 1 / np.sqrt(d))
        ref = oracle.svg2_attention_given(qh, kh, vh, aq[0, h], ak[0, h], bits[0, h])
        assert_close(f64(o[0, h]), ref, torch.bfloat16, f"svg2 call head {h}")


def test_semantic_3d_attn_video_shape_sampled():
    wl = synth.WORKLOADS["hunyuan"]
    prm = synth.SVG2_PARAMS
    q, k, v = synth.make_qkv(wl, seed=4, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, aq, ak, sel = svg.svg_semantic_3d_attn(q, k, v, wl.N, wl.F, prm["Cq"], prm["Ck"], prm["iters"], prm["p"],
                                              status=status)
    sync_ok(status)
    aq, ak = aq.cpu().numpy(), ak.cpu().numpy()
    bits = svg.selected_bits(sel, prm["Ck"])
    rows = sampled_rows(wl, n_extra=12)
    idx = torch.from_numpy(rows).to(DEV)
    scale = 1 / np.sqrt(wl.d)
    for h in (5, 20):
        qh, kh, vh = f64(q)[0, h], f64(k)[0, h], f64(v)[0, h]
        mu_q, _ = _cluster_means(qh, aq[0, h], prm["Cq"])
        mu_k, n_k = _cluster_means(kh, ak[0, h], prm["Ck"])
        _check_topp_valid(bits[0, h], mu_q, mu_k, n_k, prm["p"], scale)
        ref = oracle.svg2_attention_given(qh, kh, vh, aq[0, h], ak[0, h], bits[0, h], rows=rows)
        assert_close(f64(o[0, h, idx]), ref, torch.bfloat16, f"svg2 video head {h}")
