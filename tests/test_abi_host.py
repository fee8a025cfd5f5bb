"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

* libsvg.so loads and exports every function include/svg.h declares;
* svg_block_list (the block schedule the attention kernel walks) equals the
  oracle's brute-force tile classification of the explicit mask, bit for bit;
* argument validation rejects bad calls before anything is enqueued.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from sparse_attention_video_profile_b200 import svg

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "svg.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:SVG_API\s+)?(?:const\s+)?\w+\**\s+\**(svg_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 15
    assert sorted(svg.EXPORTED) == names
    for n in names:
        assert hasattr(svg.lib, n), n


def test_version_and_status_strings():
    assert svg.svg_abi_version() == 2
    assert svg.lib.svg_status_string(0) == b"SVG_OK"
    assert svg.lib.svg_status_string(5) == b"SVG_ERR_WORKSPACE"
    assert svg.lib.svg_status_string(99) == b"SVG_ERR_UNKNOWN"


@pytest.mark.parametrize("L,G,a", [(256, 64, 1), (2048, 256, 2), (2048, 8, 16), (700, 33, 3), (517, 50, 2),
                                   (300, 7, 100), (129, 129, 1), (1000, 1000, 1), (4000, 13, 40)])
@pytest.mark.parametrize("tile", [(128, 128), (64, 128), (128, 64), (256, 128)])
def test_block_list_matches_bruteforce(L, G, a, tile):
    Bq, Bk = tile
    kb_lo, kb_hi, f_lo, f_hi = svg.svg_block_list(L, G, a, Bq, Bk)
    active, full = oracle.block_list(oracle.banded_mask(L, G, a), Bq, Bk)
    for qb in range(active.shape[0]):
        got_a = np.zeros(active.shape[1], bool)
        got_a[kb_lo[qb]:kb_hi[qb]] = True
        got_f = np.zeros(full.shape[1], bool)
        got_f[f_lo[qb]:f_hi[qb]] = True
        np.testing.assert_array_equal(got_a, active[qb])
        np.testing.assert_array_equal(got_f, full[qb])


def test_block_list_kernel_tile_on_video_shapes():
    """At the attention kernel's own tile size, for the spatial band and the
    token-major temporal band of the two video-model shapes."""
    Bq, Bk = svg.svg_attn_tile(svg.SVG_BF16, 128)
    assert (Bq, Bk) == (128, 128)
    for (N, F, a1, a2) in ((13, 1350, 3, 181), (33, 3600, 3, 281)):
        L = N * F
        for (G, a) in ((F, a1), (N, a2)):
            kb_lo, kb_hi, f_lo, f_hi = svg.svg_block_list(L, G, a, Bq, Bk)
            # brute force on a sample of query tiles (rows of the explicit mask)
            for qb in np.linspace(0, len(kb_lo) - 1, 9).astype(int):
                rows = np.arange(qb * Bq, min(L, (qb + 1) * Bq))
                m = oracle.banded_mask(L, G, a, rows)
                nk = -(-L // Bk)
                act = np.array([m[:, kb * Bk:(kb + 1) * Bk].any() for kb in range(nk)])
                ful = np.array([m[:, kb * Bk:(kb + 1) * Bk].all() for kb in range(nk)])
                assert set(np.nonzero(act)[0]) == set(range(kb_lo[qb], kb_hi[qb]))
                assert set(np.nonzero(ful)[0]) == set(range(f_lo[qb], f_hi[qb]))


def _shape(B=1, H=2, N=4, F=64, d=64, dtype=svg.SVG_BF16):
    return svg.svg_shape(B, H, N, F, d, dtype, 0.0)


def test_validation_rejects_bad_arguments():
    s = _shape(d=96)
    p = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    st = svg.lib.svg_permute(ctypes.byref(s), p, ctypes.c_void_p(2 << 20), None, None)
    assert st == 2  # SVG_ERR_UNSUPPORTED (bf16 d = 96)
    assert b"d in {64, 128}" in svg.lib.svg_last_error()
    s = _shape()
    assert svg.lib.svg_permute(ctypes.byref(s), None, p, None, None) == 1
    assert svg.lib.svg_permute(ctypes.byref(s), ctypes.c_void_p((1 << 20) + 8), p, None, None) == 1  # misaligned
    assert svg.lib.svg_permute(ctypes.byref(s), p, p, None, None) == 1  # in place
    bad = _shape(N=0)
    assert svg.lib.svg_dense_attn(ctypes.byref(bad), p, p, p, p, None, None) == 1
    assert svg.lib.svg_block_sparse_attn(ctypes.byref(s), p, p, p, p, p, p, p, p, None, 1, 1, None, None) == 1
    assert svg.lib.svg_block_sparse_attn(ctypes.byref(s), p, p, p, p, p, p, p, p, p, 0, 1, None, None) == 1
    assert svg.lib.svg_banded_attn(ctypes.byref(s), p, p, p, p, 0, 1, None, None) == 1
    ws = ctypes.c_void_p(1 << 24)
    assert svg.lib.svg_profile_heads(ctypes.byref(s), p, p, p, 1, 1, p, 0, p, p, ws, 1 << 30, None) == 1  # S = 0
    assert svg.lib.svg_profile_heads(ctypes.byref(s), p, p, p, 1, 1, p, 129, p, p, ws, 1 << 30, None) == 1
    assert svg.lib.svg_profile_heads(ctypes.byref(s), p, p, p, 1, 1, p, 32, p, p, ws, 16, None) == 5  # workspace
    assert svg.lib.svg_block_list(0, 1, 1, 1, 1, p, p, p, p) == 1


def test_shape_struct_matches_header():
    """svg_shape as the header declares it: seven 4-byte fields, then the
    layout; a zero-initialised layout is [B, H, L, d]."""
    src = open(HEADER).read()
    body = re.search(r"typedef struct svg_shape \{(.*?)\} svg_shape;", src, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"(\w+)\s*[,;]", body)
    assert fields == ["B", "H", "N", "F", "d", "dtype", "scale", "layout"]
    assert [f for f, _ in svg.svg_shape._fields_] == fields
    assert ctypes.sizeof(svg.svg_shape) == 32 and svg.svg_shape.layout.offset == 28
    assert svg.svg_shape(1, 2, 3, 4, 64, 0, 0.0).layout == svg.SVG_LAYOUT_BHLD
    for name, val in (("SVG_LAYOUT_BHLD", 0), ("SVG_LAYOUT_BLHD", 1)):
        assert re.search(rf"#define {name} {val}\b", src)
        assert getattr(svg, name) == val


def test_layout_validation_and_sizes():
    p = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    bad = svg.svg_shape(1, 2, 4, 64, 64, svg.SVG_BF16, 0.0, 2)
    assert svg.lib.svg_permute(ctypes.byref(bad), p, ctypes.c_void_p(2 << 20), None, None) == 1
    assert b"unknown layout" in svg.lib.svg_last_error()
    assert svg.lib.svg_profile_heads_noalloc(ctypes.byref(bad), p, p, p, 1, 1, p, 16, p, p, None) == 1
    assert svg.svg_sparse_3d_attn_workspace_size(bad, 4, 16) == 0
    # the host-buffer call copies whole heads: [B, H, L, d] only
    s = svg.svg_shape(1, 2, 4, 64, 64, svg.SVG_BF16, 0.0, svg.SVG_LAYOUT_BLHD)
    st = svg.lib.svg_sparse_3d_attn_host(ctypes.byref(s), p, p, p, p, 1, 4, p, 16, p, p, 1, p, 1 << 30, None, None)
    assert st == 2 and b"[B, H, L, d]" in svg.lib.svg_last_error()
    # [B, L, H, d] whole calls always permute into [B, H, L, d] copies; the
    # tile counts and the profiling workspace do not depend on the layout
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    for (B, H, N, F, d, a2) in ((2, 3, 5, 100, 64, 60), (1, 24, 33, 3600, 128, 281), (2, 3, 16, 64, 128, 4)):
        s0 = svg.svg_shape(B, H, N, F, d, svg.SVG_BF16, 0.0, svg.SVG_LAYOUT_BHLD)
        s1 = svg.svg_shape(B, H, N, F, d, svg.SVG_BF16, 0.0, svg.SVG_LAYOUT_BLHD)
        sep0, fz0, _ = svg.svg_sparse_3d_attn_plan(s0, a2)
        sep1, fz1, fused1 = svg.svg_sparse_3d_attn_plan(s1, a2)
        assert (sep0, fz0) == (sep1, fz1) and fused1 is False
        prof = svg.svg_profile_workspace_size(s0, 64)
        assert svg.svg_profile_workspace_size(s1, 64) == prof
        assert svg.svg_sparse_3d_attn_workspace_size(s1, a2, 64) == prof + 4 * al(B * H * N * F * d * 2)
    assert svg.svg_sparse_3d_attn_plan(svg.svg_shape(1, 24, 33, 3600, 128, svg.SVG_BF16, 0.0), 281)[2] is True


def test_tf32_dtype_host_side():
    """SVG_TF32: fp32 tensors (4-byte workspaces, the fp32 profiling layout),
    128 x 128 attention tiles, d in {32, 64, 128}; the binding takes it for
    float32 tensors only."""
    import torch
    assert svg.svg_attn_tile(svg.SVG_TF32, 64) == (128, 128)
    f = svg.svg_shape(2, 3, 5, 40, 64, svg.SVG_FP32, 0.0)
    t = svg.svg_shape(2, 3, 5, 40, 64, svg.SVG_TF32, 0.0)
    assert svg.svg_profile_workspace_size(t, 32) == svg.svg_profile_workspace_size(f, 32) > 0
    assert svg.svg_sparse_3d_attn_workspace_size(t, 4, 32) == svg.svg_sparse_3d_attn_workspace_size(f, 4, 32) > 0
    assert svg.svg_workspace_size(t, 2) == svg.svg_workspace_size(f, 2)
    assert svg.svg_sparse_3d_attn_plan(t, 4)[2] is False  # fp32 tensors always permute
    p = ctypes.c_void_p(1 << 20)
    bad = svg.svg_shape(1, 2, 4, 64, 96, svg.SVG_TF32, 0.0)
    assert svg.lib.svg_dense_attn(ctypes.byref(bad), p, p, p, p, None, None) == 2
    bad = svg.svg_shape(1, 2, 4, 64, 64, 3, 0.0)
    assert svg.lib.svg_dense_attn(ctypes.byref(bad), p, p, p, p, None, None) == 1
    x = torch.empty(1, 2, 20, 64)
    assert svg.make_shape(x, 4, 5, tf32=True).dtype == svg.SVG_TF32
    with pytest.raises(TypeError):
        svg.make_shape(x.to(torch.bfloat16), 4, 5, tf32=True)


def test_make_shape_reads_either_layout():
    import torch
    x = torch.empty(2, 3, 5 * 7, 64, dtype=torch.bfloat16)  # [B, H, L, d]
    s = svg.make_shape(x, 5, 7)
    assert (s.B, s.H, s.N, s.F, s.d, s.layout) == (2, 3, 5, 7, 64, svg.SVG_LAYOUT_BHLD)
    s = svg.make_shape(x.transpose(1, 2).contiguous(), 5, 7, layout="blhd")  # [B, L, H, d]
    assert (s.B, s.H, s.N, s.F, s.d, s.layout) == (2, 3, 5, 7, 64, svg.SVG_LAYOUT_BLHD)
    with pytest.raises(ValueError):
        svg.make_shape(x, 5, 7, layout="blhd")  # 3 rows of 35 heads: L != N*F
    with pytest.raises(ValueError):
        svg.make_shape(x, 5, 7, layout="lbhd")


def test_workspace_sizes():
    s = _shape(B=1, H=24, N=33, F=3600, d=128)
    prof = svg.svg_profile_workspace_size(s, 128)
    assert prof > 0 and prof % 256 == 0
    # the whole call needs token-major copies only when it does not fuse the layout
    for shp, a2, S in [(s, 281, 128), (_shape(B=1, H=48, N=13, F=1350, d=64), 181, 128), (s, 3, 128)]:
        _, _, fused = svg.svg_sparse_3d_attn_plan(shp, a2)
        t = shp.B * shp.H * shp.N * shp.F * shp.d * 2
        extra = 0 if fused else 4 * ((t + 255) // 256 * 256)
        assert svg.svg_sparse_3d_attn_workspace_size(shp, a2, S) == svg.svg_profile_workspace_size(shp, S) + extra
    f3 = _shape(B=1, H=2, N=5, F=40, d=64, dtype=svg.SVG_FP32)
    t = 2 * 5 * 40 * 64 * 4
    t_al = (t + 255) // 256 * 256
    assert svg.svg_sparse_3d_attn_workspace_size(f3, 4, 16) == 4 * t_al + svg.svg_profile_workspace_size(f3, 16)
    assert svg.svg_sparse_3d_attn_plan(f3, 4)[2] is False  # fp32 always permutes
    assert svg.svg_profile_workspace_size(s, 0) == 0
    assert svg.svg_profile_workspace_size(s, 129) == 0
    f = _shape(dtype=svg.SVG_FP32, d=32)
    assert svg.svg_profile_workspace_size(f, 32) > 0
    # the step-by-step call: [profiling workspace at S = 128 | qp | kp | vp | op]
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    t = al(s.B * s.H * s.N * s.F * s.d * 2)
    assert svg.svg_workspace_size(s, 0) == al(prof)
    assert svg.svg_workspace_size(s, 1) == al(prof) + 4 * t
    assert svg.svg_workspace_size(s, 24) == al(prof) + 4 * t
    assert svg.svg_workspace_size(s, -1) == 0 and svg.svg_workspace_size(s, 25) == 0
    small = _shape(B=1, H=2, N=2, F=32, d=64)  # L = 64 < 128: profiling sized for S = L
    assert svg.svg_workspace_size(small, 2) == al(svg.svg_profile_workspace_size(small, 64)) + 4 * al(2 * 64 * 64 * 2)
    assert svg.svg_workspace_size(f3, 1) == al(svg.svg_profile_workspace_size(f3, 128)) + 4 * t_al


def _brute_tile_counts(N, F, a):
    """Key tiles a temporal head takes, by enumerating every CTA and every
    128-key tile and keeping the tiles holding at least one kept key of one
    of the CTA's rows (tiles between the first and the last such tile count
    too: the kernels walk one contiguous tile range per frame group)."""
    L = N * F
    # token-major copies: CTA = 256 consecutive token-major rows x' = j N + i
    sep = 0
    for q0 in range(0, L, 256):
        js = {x // N for x in range(q0, min(q0 + 256, L))}
        keys = [y for y in range(L) if any(abs(y // N - j) < a for j in (min(js), max(js)))]
        sep += keys[-1] // 128 - keys[0] // 128 + 1
    # fused: frame groups of size 2^e (largest first), a tile = 2^e frames x 128/2^e positions
    groups, left = [], N
    while left:
        s = 1
        while s * 2 <= left and s < 128:
            s *= 2
        groups.append(s)
        left -= s
    fz = 0
    for s_q in groups:
        per = 2 * 128 // s_q
        for p0 in range(0, F, per):
            pos_q = range(p0, min(p0 + per, F))
            kept = [p for p in range(F) if any(abs(p - j) < a for j in (pos_q[0], pos_q[-1]))]
            for s_k in groups:
                P = 128 // s_k
                fz += kept[-1] // P - kept[0] // P + 1
    return sep, fz


@pytest.mark.parametrize("N,F,a", [(33, 300, 20), (13, 135, 18), (4, 64, 3), (21, 100, 33), (1, 500, 7), (130, 5, 2)])
def test_layout_plan_tile_counts_match_enumeration(N, F, a):
    shp = _shape(B=1, H=1, N=N, F=F, d=64)
    sep, fz, fused = svg.svg_sparse_3d_attn_plan(shp, a)
    assert (sep, fz) == _brute_tile_counts(N, F, min(a, F))
    assert fused == (fz * 100 <= sep * 103)


def test_semantic_and_kmeans_validation_and_sizes():
    """Argument checks of the SVG2-style entry points fail before any launch
    (the pointers below are never dereferenced)."""
    s = _shape(B=1, H=2, N=4, F=100, d=128)
    f = _shape(B=1, H=2, N=4, F=100, d=64, dtype=svg.SVG_FP32)
    lib = svg.lib
    assert lib.svg_semantic_attn_workspace_size(ctypes.byref(s), 16, 64) > 0
    assert lib.svg_semantic_attn_workspace_size(ctypes.byref(f), 16, 64) == 0       # fp32
    assert lib.svg_semantic_attn_workspace_size(ctypes.byref(s), 16, 1025) == 0     # Ck > 1024
    assert lib.svg_semantic_attn_workspace_size(ctypes.byref(s), 0, 64) == 0
    assert lib.svg_kmeans_workspace_size(ctypes.byref(s), 512) > 0
    assert lib.svg_kmeans_workspace_size(ctypes.byref(s), 513) == 0                 # C > 512
    assert lib.svg_kmeans_workspace_size(ctypes.byref(f), 8) == 0
    ws3 = lib.svg_semantic_3d_attn_workspace_size(ctypes.byref(s), 16, 64)
    assert ws3 >= lib.svg_semantic_attn_workspace_size(ctypes.byref(s), 16, 64)
    assert ws3 >= lib.svg_kmeans_workspace_size(ctypes.byref(s), 64)
    p = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 24)
    big = ctypes.c_size_t(1 << 40)
    sem = lib.svg_semantic_attn
    assert sem(ctypes.byref(s), p, p, p, p, p, p, 16, 64, ctypes.c_float(0.0), p, ws, big, None, None) == 1  # p = 0
    assert sem(ctypes.byref(s), p, p, p, p, p, p, 16, 64, ctypes.c_float(1.5), p, ws, big, None, None) == 1  # p > 1
    assert sem(ctypes.byref(s), p, p, p, p, None, p, 16, 64, ctypes.c_float(0.9), p, ws, big, None, None) == 1
    assert sem(ctypes.byref(s), p, p, p, p, p, p, 16, 64, ctypes.c_float(0.9), p, ctypes.c_void_p((1 << 24) + 16),
               big, None, None) == 1  # misaligned workspace
    assert sem(ctypes.byref(s), p, p, p, p, p, p, 16, 64, ctypes.c_float(0.9), p, ws, ctypes.c_size_t(64), None,
               None) == 5  # short workspace
    assert sem(ctypes.byref(f), p, p, p, p, p, p, 16, 64, ctypes.c_float(0.9), p, ws, big, None, None) == 2  # fp32
    km = lib.svg_kmeans
    assert km(ctypes.byref(s), p, 401, 3, p, p, ws, big, None, None) == 1    # C > L (400 rows)
    assert km(ctypes.byref(s), p, 16, 0, p, p, ws, big, None, None) == 1     # iters < 1
    assert km(ctypes.byref(s), p, 16, 3, None, p, ws, big, None, None) == 1
    assert km(ctypes.byref(f), p, 16, 3, p, p, ws, big, None, None) == 2     # fp32
    fused = lib.svg_block_sparse_attn_fused
    assert fused(ctypes.byref(f), p, p, p, p, p, 1, 1, None, None) == 2      # fp32: unsupported
    assert fused(ctypes.byref(s), p, p, p, p, None, 1, 1, None, None) == 1   # no labels
    assert lib.svg_mixed_attn_fused(ctypes.byref(s), p, p, p, p, p, -1, 0, 1, None, None) == 1
