"""[B, L, H, d] tensors (SVG_LAYOUT_BLHD) against [B, H, L, d] ones.

The layout only decides where each row of d elements is read or written; the
kernels run the same arithmetic in the same order, so every entry point must
give bit-identical results on the same values in either layout (outputs
compared after moving them back to [B, H, L, d]).  Each group also checks the
[B, L, H, d] result against the fp64 oracle directly, with the tolerances of
test_gpu_parity.py.  Shapes have B = 2 (the batch stride), H = 3, ragged
sequence lengths and, for the multi-rank split, head blocks that straddle a
batch entry.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_video_profile_b200 import svg, synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-5)}


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def blhd(x):
    """[B, H, L, d] -> contiguous [B, L, H, d]."""
    return x.transpose(1, 2).contiguous()


def bhld(y):
    """[B, L, H, d] -> contiguous [B, H, L, d]."""
    return y.transpose(1, 2).contiguous()


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs = float(np.max(np.abs(got - ref)))
    rel_l2 = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    ta, tr = TOL[dtype]
    assert max_abs <= ta and rel_l2 <= tr, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel_l2:.3e}"


def workload(N, F, d, dtype="bf16", a1=2, a2=7, S=48, B=2, H=3):
    return synth.Workload(f"layout-{N}x{F}-d{d}-{dtype}", B=B, H=H, N=N, F=F, d=d, dtype=dtype, a1=a1, a2=a2,
                          S=min(S, N * F), kinds="half", weight=("const", 3.0))


def inputs(wl, seed):
    q, k, v = synth.make_qkv(wl, seed=seed, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, seed)
    return (q, k, v), (blhd(q), blhd(k), blhd(v)), rows_np, torch.from_numpy(rows_np).to(DEV)


def new_status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def sync_ok(*statuses):
    torch.cuda.synchronize()
    for s in statuses:
        assert int(s.item()) == 0, f"device status {int(s.item())}"


# ---------------------------------------------------------------- profiling

@pytest.mark.parametrize("N,F,d,dtype", [(5, 100, 64, "bf16"), (3, 301, 128, "bf16"), (4, 50, 32, "fp32")])
def test_profile_layouts_identical(N, F, d, dtype):
    wl = workload(N, F, d, dtype)
    (q, k, v), (qt, kt, vt), rows_np, rows = inputs(wl, 11)
    mse0, lab0 = svg.svg_profile_heads(q, k, v, N, F, wl.a1, wl.a2, rows)
    mse1, lab1 = svg.svg_profile_heads(qt, kt, vt, N, F, wl.a1, wl.a2, rows, layout="blhd")
    mse2, lab2 = svg.svg_profile_heads_noalloc(qt, kt, vt, N, F, wl.a1, wl.a2, rows, layout="blhd")
    torch.cuda.synchronize()
    assert torch.equal(mse0, mse1) and torch.equal(lab0, lab1)
    assert torch.equal(mse0, mse2) and torch.equal(lab0, lab2)
    ref_mse, ref_label = oracle.profile_heads(f64(q), f64(k), f64(v), N, F, wl.a1, wl.a2, rows_np)
    gap = np.abs(ref_mse[..., 0] - ref_mse[..., 1]) > 1e-3 * np.maximum(ref_mse[..., 0], ref_mse[..., 1])
    np.testing.assert_array_equal(lab1.cpu().numpy()[gap], ref_label[gap])


def test_mode_search_layouts_identical():
    wl = workload(6, 96, 128)
    (q, k, v), (qt, kt, vt), _, rows = inputs(wl, 12)
    modes = dict(window=96, md_half=8, stripe=64)
    loss0, mode0 = svg.svg_mode_search(q, k, v, wl.N, wl.F, rows, **modes)
    loss1, mode1 = svg.svg_mode_search(qt, kt, vt, wl.N, wl.F, rows, **modes, layout="blhd")
    torch.cuda.synchronize()
    assert torch.equal(loss0, loss1) and torch.equal(mode0, mode1)


# ---------------------------------------------------------------- layout transformation

@pytest.mark.parametrize("N,F,d,dtype", [(5, 37, 64, "bf16"), (7, 20, 128, "bf16"), (3, 11, 32, "fp32")])
def test_permute_layouts_identical(N, F, d, dtype):
    wl = workload(N, F, d, dtype)
    (q, k, v), (qt, kt, vt), _, _ = inputs(wl, 13)
    label = torch.tensor([[1, 0, 1], [0, 1, 1]], dtype=torch.int8, device=DEV)
    fill = 7.0
    outs0 = tuple(torch.full_like(x, fill) for x in (q, k, v))
    outs1 = tuple(torch.full_like(x, fill) for x in (qt, kt, vt))
    qp0, kp0, vp0 = svg.svg_permute_qkv(q, k, v, N, F, label, out=outs0)
    qp1, kp1, vp1 = svg.svg_permute_qkv(qt, kt, vt, N, F, label, out=outs1, layout="blhd")
    back1 = svg.svg_unpermute(qp1, N, F, label, out=torch.full_like(qt, fill), layout="blhd")
    torch.cuda.synchronize()
    for a, b in ((qp0, qp1), (kp0, kp1), (vp0, vp1)):
        assert torch.equal(a, bhld(b))  # moved heads permuted, the others untouched (still `fill`)
    # temporal heads back in frame-major order, spatial heads untouched by both passes
    ref = oracle.permute(f64(q), N, F)
    qp1n, back1n = f64(bhld(qp1)), f64(bhld(back1))
    for b in range(2):
        for h in range(3):
            if label[b, h] == 1:
                np.testing.assert_array_equal(qp1n[b, h], ref[b, h])
                np.testing.assert_array_equal(back1n[b, h], f64(q)[b, h])
            else:
                assert np.all(qp1n[b, h] == fill) and np.all(back1n[b, h] == fill)


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("N,F,d", [(5, 100, 64), (4, 130, 128)])
def test_block_sparse_layouts_identical(N, F, d):
    wl = workload(N, F, d, a1=2, a2=9)
    (q, k, v), (qt, kt, vt), _, _ = inputs(wl, 14)
    label = torch.tensor([[1, 0, 1], [0, 1, 0]], dtype=torch.int8, device=DEV)
    s0, s1, s2, s3 = new_status(), new_status(), new_status(), new_status()
    qp0, kp0, vp0 = svg.svg_permute_qkv(q, k, v, N, F, label)
    qp1, kp1, vp1 = svg.svg_permute_qkv(qt, kt, vt, N, F, label, layout="blhd")
    o0, op0 = svg.svg_block_sparse_attn(q, k, v, qp0, kp0, vp0, label, N, F, wl.a1, wl.a2, status=s0)
    o1, op1 = svg.svg_block_sparse_attn(qt, kt, vt, qp1, kp1, vp1, label, N, F, wl.a1, wl.a2, status=s1,
                                        layout="blhd")
    f0 = svg.svg_block_sparse_attn_fused(q, k, v, label, N, F, wl.a1, wl.a2, status=s2)
    f1 = svg.svg_block_sparse_attn_fused(qt, kt, vt, label, N, F, wl.a1, wl.a2, status=s3, layout="blhd")
    sync_ok(s0, s1, s2, s3)
    lab = label.cpu().numpy()
    o0c, o1c, op0c, op1c = o0.cpu(), bhld(o1).cpu(), op0.cpu(), bhld(op1).cpu()
    for b in range(2):
        for h in range(3):
            if lab[b, h] == 0:
                assert torch.equal(o0c[b, h], o1c[b, h])
            else:
                assert torch.equal(op0c[b, h], op1c[b, h])
    assert torch.equal(f0, bhld(f1))
    ref = oracle.sparse_attention(f64(q), f64(k), f64(v), lab, N, F, wl.a1, wl.a2)
    assert_close(f64(bhld(f1)), ref, torch.bfloat16, "fused, [B, L, H, d]")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64)])
def test_dense_layouts_identical(dtype, d):
    wl = workload(3, 70, d, dtype)
    (q, k, v), (qt, kt, vt), _, _ = inputs(wl, 15)
    o0 = svg.svg_dense_attn(q, k, v, wl.N, wl.F)
    o1 = svg.svg_dense_attn(qt, kt, vt, wl.N, wl.F, layout="blhd")
    torch.cuda.synchronize()
    assert torch.equal(o0, bhld(o1))
    assert_close(f64(bhld(o1)), oracle.dense_attention(f64(q), f64(k), f64(v)), q.dtype, "dense, [B, L, H, d]")


def separate_call(q, k, v, N, F, a1, a2, rows, status):
    """The whole call's separate plan on [B, H, L, d] tensors, step by step:
    profile -> permute -> block-sparse attention -> unpermute (the plan the
    [B, L, H, d] whole call always takes)."""
    mse, label = svg.svg_profile_heads(q, k, v, N, F, a1, a2, rows)
    qp, kp, vp = svg.svg_permute_qkv(q, k, v, N, F, label)
    o, op = svg.svg_block_sparse_attn(q, k, v, qp, kp, vp, label, N, F, a1, a2, status=status)
    svg.svg_unpermute(op, N, F, label, out=o)
    return o, mse, label


def test_whole_call_plan_by_layout():
    """[B, L, H, d] whole calls permute into copies; [B, H, L, d] ones fuse
    where the fused tiling costs little (both plans occur in the shapes below)."""
    plans = set()
    for (N, F, a2) in WHOLE_CALL_SHAPES:
        s0 = svg.svg_shape(2, 3, N, F, 64, svg.SVG_BF16, 0.0, svg.SVG_LAYOUT_BHLD)
        s1 = svg.svg_shape(2, 3, N, F, 64, svg.SVG_BF16, 0.0, svg.SVG_LAYOUT_BLHD)
        plans.add(svg.svg_sparse_3d_attn_plan(s0, a2)[2])
        assert svg.svg_sparse_3d_attn_plan(s1, a2)[2] is False
    assert plans == {True, False}


WHOLE_CALL_SHAPES = ((16, 64, 4), (5, 100, 60), (8, 128, 3), (3, 200, 150))


@pytest.mark.parametrize("N,F,a2", WHOLE_CALL_SHAPES)
@pytest.mark.parametrize("d", [64, 128])
def test_whole_call_layouts_identical(N, F, a2, d):
    wl = workload(N, F, d, a1=2, a2=a2)
    (q, k, v), (qt, kt, vt), rows_np, rows = inputs(wl, 16)
    s0, s1 = new_status(), new_status()
    o0, mse0, lab0 = separate_call(q, k, v, N, F, wl.a1, wl.a2, rows, s0)
    o1, mse1, lab1 = svg.svg_sparse_3d_attn(qt, kt, vt, N, F, wl.a1, wl.a2, rows, status=s1, layout="blhd")
    sync_ok(s0, s1)
    assert torch.equal(mse0, mse1) and torch.equal(lab0, lab1)
    assert torch.equal(o0, bhld(o1))
    ref = oracle.sparse_attention(f64(q), f64(k), f64(v), lab1.cpu().numpy(), N, F, wl.a1, wl.a2)
    assert_close(f64(bhld(o1)), ref, torch.bfloat16, "whole call, [B, L, H, d]")


def test_whole_call_fp32_layouts_identical():
    wl = workload(4, 40, 32, "fp32", a1=1, a2=5, S=32)
    (q, k, v), (qt, kt, vt), _, rows = inputs(wl, 17)
    o0, mse0, lab0 = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows)
    o1, mse1, lab1 = svg.svg_sparse_3d_attn(qt, kt, vt, wl.N, wl.F, wl.a1, wl.a2, rows, layout="blhd")
    torch.cuda.synchronize()
    assert torch.equal(mse0, mse1) and torch.equal(lab0, lab1) and torch.equal(o0, bhld(o1))
    ref = oracle.sparse_attention(f64(q), f64(k), f64(v), lab1.cpu().numpy(), wl.N, wl.F, wl.a1, wl.a2)
    assert_close(f64(bhld(o1)), ref, torch.float32, "fp32 whole call")


def test_mixed_layouts_identical():
    wl = workload(6, 80, 128)
    (q, k, v), (qt, kt, vt), _, _ = inputs(wl, 18)
    mode = torch.tensor([[0, 2, 3], [4, 1, 3]], dtype=torch.int8, device=DEV)
    prm = dict(window=80, md_half=6, stripe=100)
    o0 = svg.svg_mixed_3d_attn(q, k, v, mode, wl.N, wl.F, **prm)
    o1 = svg.svg_mixed_3d_attn(qt, kt, vt, mode, wl.N, wl.F, **prm, layout="blhd")
    f0 = svg.svg_mixed_attn_fused(q, k, v, mode, wl.N, wl.F, **prm)
    f1 = svg.svg_mixed_attn_fused(qt, kt, vt, mode, wl.N, wl.F, **prm, layout="blhd")
    torch.cuda.synchronize()
    assert torch.equal(o0, bhld(o1)) and torch.equal(f0, bhld(f1))
    ref = oracle.mixed_attention(f64(q), f64(k), f64(v), mode.cpu().numpy(), wl.N, wl.F, **prm)
    assert_close(f64(bhld(o1)), ref, torch.bfloat16, "mixed, [B, L, H, d]")


def test_svg2_layouts_identical():
    wl = workload(4, 250, 128)
    (q, k, v), (qt, kt, vt), _, _ = inputs(wl, 19)
    Cq, Ck, iters, p = 16, 32, 3, 0.9
    s0, s1 = new_status(), new_status()
    r0 = svg.svg_semantic_3d_attn(q, k, v, wl.N, wl.F, Cq, Ck, iters, p, status=s0)
    r1 = svg.svg_semantic_3d_attn(qt, kt, vt, wl.N, wl.F, Cq, Ck, iters, p, status=s1, layout="blhd")
    sync_ok(s0, s1)
    o0, aq0, ak0, sel0 = r0
    o1, aq1, ak1, sel1 = r1
    assert torch.equal(aq0, aq1) and torch.equal(ak0, ak1) and torch.equal(sel0, sel1)
    assert torch.equal(o0, bhld(o1))
    qn, kn, vn, on = f64(q), f64(k), f64(v), f64(bhld(o1))
    aq, ak, bits = aq1.cpu().numpy(), ak1.cpu().numpy(), svg.selected_bits(sel1, Ck)
    for b in range(2):
        for h in range(3):
            ref = oracle.svg2_attention_given(qn[b, h], kn[b, h], vn[b, h], aq[b, h], ak[b, h], bits[b, h])
            assert_close(on[b, h], ref, torch.bfloat16, f"SVG2, [B, L, H, d], head ({b}, {h})")


# ---------------------------------------------------------------- head blocks of one call

@pytest.mark.parametrize("world", [2, 4])
def test_shard_layouts_identical(world):
    """Each rank's block of heads, one rank after another on one GPU; with
    world = 4 the second block holds the last head of batch entry 0 and the
    first of batch entry 1.  Outputs and labels equal the single whole call;
    the MSEs equal the [B, H, L, d] shards' (the key split of profiling
    depends on the block's head count)."""
    wl = workload(5, 100, 128, a1=2, a2=60)
    (q, k, v), (qt, kt, vt), _, rows = inputs(wl, 20)
    full, _, lab_full = svg.svg_sparse_3d_attn(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows)
    res = {}
    status = new_status()
    for layout, (a, b, c) in (("bhld", (q, k, v)), ("blhd", (qt, kt, vt))):
        o = torch.zeros_like(a)
        mse = torch.zeros(2, 3, 2, dtype=torch.float32, device=DEV)
        label = torch.full((2, 3), -1, dtype=torch.int8, device=DEV)
        for rank in range(world):  # independent calls, one after the other
            svg.svg_sparse_3d_attn_shard(a, b, c, wl.N, wl.F, wl.a1, wl.a2, rows, rank, world, o=o, mse=mse,
                                         label=label, status=status, layout=layout)
        res[layout] = (o if layout == "bhld" else bhld(o), mse, label)
    sync_ok(status)
    (o0, mse0, lab0), (o1, mse1, lab1) = res["bhld"], res["blhd"]
    assert torch.equal(mse0, mse1) and torch.equal(lab0, lab1) and torch.equal(o0, o1)
    assert torch.equal(lab1, lab_full) and torch.equal(o1, full)


# ---------------------------------------------------------------- video-model shapes

@pytest.mark.parametrize("name", ["cogvideox", "hunyuan"])
def test_video_shape_layouts_identical(name):
    """The full call at the video-model shape, every output element: the
    [B, L, H, d] whole call against the same plan on [B, H, L, d] tensors,
    and the fused attention in both layouts."""
    wl = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(wl, seed=3, device=DEV)
    rows = torch.from_numpy(synth.sample_rows(wl.L, wl.S, 3)).to(DEV)
    s0, s1, s2, s3 = new_status(), new_status(), new_status(), new_status()
    o0, mse0, lab0 = separate_call(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows, s0)
    f0 = svg.svg_block_sparse_attn_fused(q, k, v, lab0, wl.N, wl.F, wl.a1, wl.a2, status=s2)
    torch.cuda.synchronize()
    o0, f0 = o0.cpu(), f0.cpu()
    qt, kt, vt = blhd(q), blhd(k), blhd(v)
    del q, k, v
    torch.cuda.empty_cache()
    o1, mse1, lab1 = svg.svg_sparse_3d_attn(qt, kt, vt, wl.N, wl.F, wl.a1, wl.a2, rows, status=s1, layout="blhd")
    f1 = svg.svg_block_sparse_attn_fused(qt, kt, vt, lab1, wl.N, wl.F, wl.a1, wl.a2, status=s3, layout="blhd")
    sync_ok(s0, s1, s2, s3)
    assert torch.equal(mse0, mse1) and torch.equal(lab0, lab1)
    assert torch.equal(o0, bhld(o1).cpu())
    assert torch.equal(f0, bhld(f1).cpu())
