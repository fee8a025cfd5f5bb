"""fp32 tensors through the tensor cores in tf32 (SVG_TF32) against the oracle.

Two bars:
* against the fp64 oracle (the method's definition on the given fp32
  inputs): max-abs 1e-2 and relative L2 4e-3.  tf32 keeps 10 of fp32's 23
  mantissa bits, so each input element carries a relative error of up to
  2^-10; an fp64 emulation of that truncation (the helper below) reaches
  4.1e-3 max-abs and 1.3e-3 relative L2 on these shapes, and the bars are
  about twice that;
* against that emulation itself (Q, K, V cut to tf32; the keys taken 128 at
  a time with a running maximum, each tile's weights rounded to nearest tf32
  against the maximum so far; everything else exact): max-abs 5e-4 and
  relative L2 5e-5.  A weight that falls on the other side of a tf32 rounding
  boundary in the kernel's fp32 than in the emulation's fp64 moves an output
  element by up to 2^-11 |v| (the max-abs bar); rounding the inputs to
  nearest instead of cutting them misses the relative bar by more than an
  order of magnitude, so it shows the kernel computes tf32 attention as
  stated and nothing cruder.
Labels come from the fp32 profiling path and must equal SVG_FP32's.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_video_profile_b200 import svg, synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ORACLE_TOL = (1e-2, 4e-3)
EMUL_TOL = (5e-4, 5e-5)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def close(got, ref, tol, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs = float(np.max(np.abs(got - ref)))
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= tol[0] and rel <= tol[1], f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"
    return max_abs, rel


def tf32_cut(x):
    """fp32 values with the low 13 mantissa bits cleared (what a tf32 operand keeps)."""
    a = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return a.view(np.float32).astype(np.float64)


def tf32_round(x):
    """Round to the nearest tf32 value, ties away from zero (fp32 in, fp64 out)."""
    a = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    a = (a + 0x1000) & 0xFFFFE000
    return a.astype(np.uint32).view(np.float32).astype(np.float64)


def emulate(q, k, v, mask, scale, tile=128):
    """One head of banded attention in tf32 arithmetic, otherwise exact: the
    keys in tiles of 128 with a running row maximum, each tile's weights
    rounded to tf32 against the maximum so far, earlier sums rescaled."""
    s = (tf32_cut(q) @ tf32_cut(k).T) * scale * np.log2(np.e)
    s = np.where(mask, s, -np.inf)
    vt = tf32_cut(v)
    R, L = s.shape
    m = np.full((R, 1), -np.inf)
    acc = np.zeros((R, vt.shape[1]))
    l = np.zeros((R, 1))
    for y0 in range(0, L, tile):
        st = s[:, y0:y0 + tile]
        m_new = np.maximum(m, st.max(axis=1, keepdims=True))
        with np.errstate(invalid="ignore"):
            alpha = np.where(np.isneginf(m_new), 1.0, np.exp2(m - m_new))
            p = np.where(np.isneginf(m_new), 0.0, np.exp2(st - m_new))
        p = tf32_round(p.astype(np.float32))
        acc = acc * alpha + p @ vt[y0:y0 + tile]
        l = l * alpha + p.sum(axis=1, keepdims=True)
        m = m_new
    return acc / l


def rand_qkv(B, H, L, d, seed, std=1.0):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return tuple((torch.randn(B, H, L, d, generator=g, device=DEV) * std).contiguous() for _ in range(3))


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("L", [60, 128, 129, 300])
def test_tf32_dense(d, L):
    q, k, v = rand_qkv(1, 2, L, d, seed=L + d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_dense_attn(q, k, v, 1, L, status=status, tf32=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    qn, kn, vn, on = f64(q), f64(k), f64(v), f64(o)
    close(on, oracle.dense_attention(qn, kn, vn), ORACLE_TOL, f"dense d={d} L={L}")
    mask = np.ones((L, L), bool)
    for h in range(2):
        em = emulate(q[0, h].cpu().numpy(), k[0, h].cpu().numpy(), v[0, h].cpu().numpy(), mask, d ** -0.5)
        close(on[0, h], em, EMUL_TOL, f"dense d={d} L={L} head {h} vs tf32 emulation")


@pytest.mark.parametrize("G,a", [(50, 1), (50, 2), (7, 3), (256, 1)])
def test_tf32_banded(G, a):
    L, d = 400, 64
    q, k, v = rand_qkv(2, 2, L, d, seed=G * 10 + a)
    o = svg.svg_banded_attn(q, k, v, 1, L, G, a, tf32=True)
    torch.cuda.synchronize()
    mask = oracle.banded_mask(L, G, a)
    ref = np.stack([[oracle.attention(f64(q)[b, h], f64(k)[b, h], f64(v)[b, h], mask) for h in range(2)]
                    for b in range(2)])
    close(f64(o), ref, ORACLE_TOL, f"banded G={G} a={a}")
    em = emulate(q[1, 1].cpu().numpy(), k[1, 1].cpu().numpy(), v[1, 1].cpu().numpy(), mask, d ** -0.5)
    close(f64(o)[1, 1], em, EMUL_TOL, "banded vs tf32 emulation")


@pytest.mark.parametrize("N,F,d", [(4, 64, 64), (5, 37, 32), (3, 100, 128)])
def test_tf32_whole_call(N, F, d):
    """The tiny workload's recipe at three shapes: labels as the fp32 call,
    output within the tf32 bar of the oracle under those labels."""
    wl = synth.Workload(f"tf32-{N}x{F}-d{d}", B=1, H=2, N=N, F=F, d=d, dtype="fp32", a1=1, a2=4,
                        S=min(32, N * F), kinds="fixed01", weight=("const", 3.0))
    q, k, v = synth.make_qkv(wl, seed=1, device=DEV)
    rows = torch.from_numpy(synth.sample_rows(wl.L, wl.S, 1)).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o32, mse32, lab32 = svg.svg_sparse_3d_attn(q, k, v, N, F, wl.a1, wl.a2, rows)
    o, mse, lab = svg.svg_sparse_3d_attn(q, k, v, N, F, wl.a1, wl.a2, rows, status=status, tf32=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(lab, lab32) and torch.equal(mse, mse32)
    ref = oracle.sparse_attention(f64(q), f64(k), f64(v), lab.cpu().numpy(), N, F, wl.a1, wl.a2)
    close(f64(o), ref, ORACLE_TOL, "whole call, tf32")
    assert not torch.equal(o, o32)  # the tensor cores ran: tf32 products differ from the fp32 path's


def test_tf32_block_sparse_with_labels():
    N, F, d = 6, 50, 64
    q, k, v = rand_qkv(2, 3, N * F, d, seed=5, std=0.7)
    label = torch.tensor([[1, 0, 1], [0, 1, 1]], dtype=torch.int8, device=DEV)
    qp, kp, vp = svg.svg_permute_qkv(q, k, v, N, F, label)
    o, op = svg.svg_block_sparse_attn(q, k, v, qp, kp, vp, label, N, F, 2, 9, tf32=True)
    o = svg.svg_unpermute(op, N, F, label, out=o)
    torch.cuda.synchronize()
    ref = oracle.sparse_attention(f64(q), f64(k), f64(v), label.cpu().numpy(), N, F, 2, 9)
    close(f64(o), ref, ORACLE_TOL, "block-sparse, tf32")


def test_tf32_layouts_identical():
    N, F, d = 5, 60, 128
    q, k, v = rand_qkv(2, 3, N * F, d, seed=6)
    rows = torch.from_numpy(synth.sample_rows(N * F, 40, 6)).to(DEV)
    o0, mse0, lab0 = svg.svg_sparse_3d_attn(q, k, v, N, F, 2, 9, rows, tf32=True)
    qt, kt, vt = (t.transpose(1, 2).contiguous() for t in (q, k, v))
    o1, mse1, lab1 = svg.svg_sparse_3d_attn(qt, kt, vt, N, F, 2, 9, rows, tf32=True, layout="blhd")
    torch.cuda.synchronize()
    assert torch.equal(mse0, mse1) and torch.equal(lab0, lab1)
    assert torch.equal(o0, o1.transpose(1, 2))
