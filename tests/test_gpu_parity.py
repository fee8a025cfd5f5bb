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
are compared as root-mean-square distances: by the triangle inequality
|sqrt(mse_gpu) - sqrt(mse_oracle)| is at most the RMS error of the two
outputs it compares, which the attention tolerance bounds by about 1e-2 for
bf16 (1e-5 for fp32).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_video_profile_b200 import svg, synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-5)}
RMS_TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-5}


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

def check_profile(mse, label, ref_mse, ref_label, dtype):
    mse = mse.cpu().numpy().astype(np.float64)
    label = label.cpu().numpy()
    gap = np.abs(ref_mse[..., 0] - ref_mse[..., 1]) / np.maximum(ref_mse.max(-1), 1e-300)
    decided = gap > 1e-3
    np.testing.assert_array_equal(label[decided], ref_label[decided])
    assert np.all(np.isin(label, [0, 1]))
    dist = np.abs(np.sqrt(mse) - np.sqrt(ref_mse))
    assert dist.max() <= RMS_TOL[dtype], f"rms distance {dist.max():.3e}"


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_profile_synthetic(name):
    wl = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(wl, seed=0, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, 0)
    rows = torch.from_numpy(rows_np).to(DEV)
    mse, label = svg.svg_profile_heads(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows)
    sync_ok()
    ref_mse, ref_label = oracle.profile_heads(f64(q), f64(k), f64(v), wl.N, wl.F, wl.a1, wl.a2, rows_np)
    check_profile(mse, label, ref_mse, ref_label, q.dtype)
    np.testing.assert_array_equal(label.cpu().numpy(), synth.head_kinds(wl, 0))


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
    ref_mse, ref_label = oracle.profile_heads(f64(q), f64(k), f64(v), N, F, a1, a2, rows_np)
    check_profile(mse, label, ref_mse, ref_label, dtype)


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
    check_profile(mse, label, ref_mse, ref_label, q.dtype)
    ref = oracle.sparse_attention(qn, kn, vn, label.cpu().numpy(), wl.N, wl.F, wl.a1, wl.a2)
    assert_close(f64(o), ref, q.dtype, name)


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
                      ref_mse, ref_label, q.dtype)
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
                      ref_mse, ref_label, q.dtype)
        ref = oracle.sparse_attention(qn, kn, vn, label_np[:, h:h + 1], wl.N, wl.F, wl.a1, wl.a2, rows=check_rows)
        got = f64(o[:, h:h + 1, torch.from_numpy(check_rows).to(DEV)])
        assert_close(got, ref, q.dtype, f"density {density} head {h}")


# ---------------------------------------------------------------- failure detection

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

def check_mode_search(loss, mode, ref_loss, ref_mode, sp, lam, eps):
    """Losses as RMS distances of their MSE parts (tolerance as for the
    profiling MSEs); modes equal wherever the oracle's decision has a margin
    larger than the MSE error that tolerance allows."""
    loss = loss.cpu().numpy().astype(np.float64)
    mode = mode.cpu().numpy()
    assert np.all(np.isfinite(loss))
    pen = lam * (1.0 - np.asarray(sp))
    mse, ref_mse = np.maximum(loss - pen, 0.0), ref_loss - pen
    dist = np.abs(np.sqrt(mse) - np.sqrt(ref_mse))
    assert dist.max() <= RMS_TOL[torch.bfloat16], f"rms distance {dist.max():.3e}"
    delta = RMS_TOL[torch.bfloat16]
    err = delta * (2 * np.sqrt(ref_mse.max(-1)) + delta)  # bound on |mse_gpu - mse_ref|
    srt = np.sort(ref_loss, -1)
    decided = (srt[..., 1] - srt[..., 0] > 2 * err) & (np.abs(srt[..., 0] - eps) > err)
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
    check_mode_search(loss, mode, ref_loss, ref_mode, sp, 0.5, 1.0)
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
    for lam, eps in [(0.5, 1.0), (0.05, 0.3)]:
        loss, mode = svg.svg_mode_search(q, k, v, N, F, rows, W, h, P, lam=lam, epsilon=eps)
        sync_ok()
        ref_loss, ref_mode = oracle.mode_search(f64(q), f64(k), f64(v), N, F, rows_np, W, h, P, lam=lam, eps=eps)
        sp = [oracle.mode_sparsity(m, N, F, W, h, P) for m in oracle.SEARCH_MODES]
        check_mode_search(loss, mode, ref_loss, ref_mode, sp, lam, eps)


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
    decided = check_mode_search(loss, mode, ref_loss, ref_mode, sp, 0.5, 1.0)
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


@pytest.mark.parametrize("d,C", [(128, 40), (64, 300), (128, 512)])
def test_kmeans_one_round_and_several(d, C):
    N, F, H = 3, 700, 2
    q, _, _ = rand_qkv(1, H, N * F, d, torch.bfloat16, 90 + C)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    a1, mu1 = svg.svg_kmeans(q, N, F, C, 1, status=status)
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
        # five rounds: close to the oracle's objective from the same start
        g5 = a5.cpu().numpy()[0, h]
        obj_gpu = oracle.kmeans_objective(x, _cluster_means(x, g5, C)[0], g5)
        ga, gmu, _ = oracle.kmeans(x, C, 5)
        obj_ref = oracle.kmeans_objective(x, gmu, ga)
        assert abs(obj_gpu - obj_ref) <= 0.02 * obj_ref, (obj_gpu, obj_ref)


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
    for h in (5, 20):
        qh, kh, vh = f64(q)[0, h], f64(k)[0, h], f64(v)[0, h]
        ref = oracle.svg2_attention_given(qh, kh, vh, aq[0, h], ak[0, h], bits[0, h], rows=rows)
        assert_close(f64(o[0, h, idx]), ref, torch.bfloat16, f"svg2 video head {h}")
