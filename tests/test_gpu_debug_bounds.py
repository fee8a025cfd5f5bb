"""The range-checked build (libsvg_debug.so, svg_debug_checks() == 1) on the
tiny and small shapes: every tensor-core kernel path -- banded and fused
attention, mixed patterns, the SVG2 cluster-pair mode, k-means, profiling,
the tf32 attention of fp32 tensors --
runs with its global indices checked, and must report no SVG_DEV_BOUNDS and
still match the fp64 oracle.  This stands in for a memory checker: an index
outside its buffer is recorded in the status word and the access skipped,
so nothing faults.

The checked library is loaded as a second instance of the binding module
(SVG_LIB names the library at import), beside the normal one.
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_video_profile_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
PKG = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "sparse_attention_video_profile_b200")
BF16_TOL = (2e-2, 1e-2)


@pytest.fixture(scope="module")
def dsvg():
    path = os.path.join(PKG, "libsvg_debug.so")
    assert os.path.exists(path), "libsvg_debug.so is not built (python -m sparse_attention_video_profile_b200.build --debug)"
    spec = importlib.util.spec_from_file_location("svg_checked", os.path.join(PKG, "svg.py"))
    mod = importlib.util.module_from_spec(spec)
    old = os.environ.get("SVG_LIB")
    os.environ["SVG_LIB"] = path
    try:
        spec.loader.exec_module(mod)
    finally:
        if old is None:
            del os.environ["SVG_LIB"]
        else:
            os.environ["SVG_LIB"] = old
    assert mod.lib.svg_debug_checks() == 1
    return mod


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def close(got, ref, what):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    max_abs = float(np.max(np.abs(got - ref)))
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= BF16_TOL[0] and rel <= BF16_TOL[1], f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


def no_bounds(status, what):
    torch.cuda.synchronize()
    st = int(status.item())
    assert st == 0, f"{what}: status word {st:#x} (SVG_DEV_BOUNDS = 0x4)"


def rand_qkv(B, H, L, d, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return tuple(torch.randn(B, H, L, d, generator=g, device=DEV).to(torch.bfloat16) for _ in range(3))


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_whole_call_checked(dsvg, name):
    wl = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(wl, seed=1, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, 1)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, mse, label = dsvg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, torch.from_numpy(rows_np).to(DEV),
                                            status=status)
    no_bounds(status, name)
    qn, kn, vn = f64(q), f64(k), f64(v)
    _, ref_label = oracle.profile_heads(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np)
    np.testing.assert_array_equal(label.cpu().numpy(), ref_label)
    ref = oracle.sparse_attention(qn, kn, vn, label.cpu().numpy(), wl.N, wl.F, wl.a1, wl.a2)
    got = f64(o)
    if q.dtype == torch.float32:
        assert np.max(np.abs(got - ref)) <= 1e-4
    else:
        close(got, ref, name)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,F,G,a", [(3, 100, 100, 1), (3, 100, 3, 5), (2, 40, 80, 1), (5, 61, 1, 1), (6, 300, 6, 1000)])
def test_banded_checked(dsvg, d, N, F, G, a):
    L = N * F
    q, k, v = rand_qkv(1, 2, L, d, 2)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = dsvg.svg_banded_attn(q, k, v, N, F, G, a, status=status)
    no_bounds(status, "banded")
    mask = oracle.banded_mask(L, min(G, L), a)
    for h in range(2):
        close(f64(o)[0, h], oracle.attention(f64(q)[0, h], f64(k)[0, h], f64(v)[0, h], mask), f"head {h}")


@pytest.mark.parametrize("N,F,d", [(6, 90, 128), (33, 17, 128), (7, 1, 64), (130, 3, 64), (13, 45, 64)])
def test_fused_checked(dsvg, N, F, d):
    q, k, v = rand_qkv(2, 4, N * F, d, 50 + N)
    label = torch.tensor([[1, 0, 1, 1], [0, 1, 0, 1]], dtype=torch.int8, device=DEV)
    a1, a2 = min(2, N), max(1, min(F, 7))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = dsvg.svg_block_sparse_attn_fused(q, k, v, label, N, F, a1, a2, status=status)
    no_bounds(status, "fused")
    close(f64(o), oracle.sparse_attention(f64(q), f64(k), f64(v), label.cpu().numpy(), N, F, a1, a2), "fused")


@pytest.mark.parametrize("fused", [False, True])
def test_mixed_checked(dsvg, fused):
    N, F = 6, 90
    modes_np = np.array([[0, 1, 2, 3, 4, 3, 3, 4, 0, 2]], dtype=np.int8)
    q, k, v = rand_qkv(1, 10, N * F, 128, 61)
    mode = torch.from_numpy(modes_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    if fused:
        o = dsvg.svg_mixed_attn_fused(q, k, v, mode, N, F, F, 7, 100, status=status)
    else:
        o = dsvg.svg_mixed_3d_attn(q, k, v, mode, N, F, F, 7, 100, status=status)
    no_bounds(status, "mixed")
    close(f64(o), oracle.mixed_attention(f64(q), f64(k), f64(v), modes_np, N, F, F, 7, 100), "mixed")


@pytest.mark.parametrize("d", [64, 128])
def test_svg2_and_kmeans_checked(dsvg, d):
    N, F, Cq, Ck, p = 4, 300, 10, 40, 0.9
    q, k, v = rand_qkv(1, 2, N * F, d, 95)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, aq, ak, sel = dsvg.svg_semantic_3d_attn(q, k, v, N, F, Cq, Ck, 3, p, status=status)
    no_bounds(status, "svg2")
    aq, ak = aq.cpu().numpy(), ak.cpu().numpy()
    assert aq.min() >= 0 and aq.max() < Cq and ak.min() >= 0 and ak.max() < Ck
    bits = dsvg.selected_bits(sel, Ck)
    for h in range(2):
        ref = oracle.svg2_attention_given(f64(q)[0, h], f64(k)[0, h], f64(v)[0, h], aq[0, h], ak[0, h], bits[0, h])
        close(f64(o[0, h]), ref, f"svg2 head {h}")


def test_profile_and_mode_search_checked(dsvg):
    wl = synth.WORKLOADS["small"]
    q, k, v = synth.make_qkv(wl, seed=4, device=DEV)
    rows = torch.from_numpy(synth.sample_rows(wl.L, wl.S, 4)).to(DEV)
    # profiling's own status word lives in its workspace: a checked-build
    # failure there shows as labels -1 and NaN MSEs
    mse, label = dsvg.svg_profile_heads(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows)
    loss, mode = dsvg.svg_mode_search(q, k, v, wl.N, wl.F, rows, wl.F, 7, 100)
    torch.cuda.synchronize()
    assert torch.all(label >= 0) and torch.all(torch.isfinite(mse))
    assert torch.all(mode >= 0) and torch.all(torch.isfinite(loss))
    np.testing.assert_array_equal(label.cpu().numpy(), synth.head_kinds(wl, 4))


@pytest.mark.parametrize("d", [32, 128])
def test_tf32_checked(dsvg, d):
    """fp32 tensors in tf32, with labels (token-major copies) and ragged L."""
    N, F = 5, 61
    g = torch.Generator(device=DEV)
    g.manual_seed(70 + d)
    q, k, v = (torch.randn(2, 3, N * F, d, generator=g, device=DEV) for _ in range(3))
    rows = torch.from_numpy(synth.sample_rows(N * F, 32, 7)).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, mse, label = dsvg.svg_sparse_3d_attn(q, k, v, N, F, 2, 9, rows, status=status, tf32=True)
    no_bounds(status, "tf32")
    ref = oracle.sparse_attention(f64(q), f64(k), f64(v), label.cpu().numpy(), N, F, 2, 9)
    got = f64(o)
    assert np.max(np.abs(got - ref)) <= 1e-2 and np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 4e-3
