"""The allocation-free profiling entry point, svg_profile_heads_noalloc.

It exists for callers that cannot allocate device memory: a plugin handed
only its input and output tensors, or a loop that must not call cudaMalloc
because that call can synchronise the whole device.  It uses the library's
fixed scratch array instead of a workspace.

This test calls it straight through the C ABI (ctypes, raw device pointers),
twice in a row on the same inputs.  It compares the results with the fp64
oracle and with svg_profile_heads, which uses a caller workspace, within the
profiling tolerance of the other GPU tests (a bound derived from the kernels'
rounding), and checks that a shape too large for the array is refused.  The
file is named to be collected last, so a run that stops at the first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mse_bound import mse_error_bounds
from sparse_attention_video_profile_b200 import svg, synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bounds(q, k, v, wl, rows_np):
    """[B, H, 2] rounding bounds of the profiling MSEs (as in the parity tests)."""
    qn, kn, vn = (t.to("cpu", torch.float64).numpy() for t in (q, k, v))
    masks = [oracle.spatial_mask(wl.N, wl.F, wl.a1, rows=rows_np), oracle.temporal_mask(wl.N, wl.F, wl.a2, rows=rows_np)]
    out = np.zeros((wl.B, wl.H, 2))
    for b in range(wl.B):
        for h in range(wl.H):
            out[b, h] = mse_error_bounds(qn[b, h], kn[b, h], vn[b, h], rows_np, masks)[0]
    return out


def _noalloc_raw(q, k, v, N, F, a1, a2, rows, mse, label):
    shape = svg.make_shape(q, N, F)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return svg.lib.svg_profile_heads_noalloc(
        ctypes.byref(shape), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), a1, a2, ctypes.c_void_p(rows.data_ptr()), rows.numel(),
        ctypes.c_void_p(mse.data_ptr()), ctypes.c_void_p(label.data_ptr()), stream)


def _check_against_workspace_version(wl, seed, H=None, against_oracle=False):
    if H is not None:
        import dataclasses
        wl = dataclasses.replace(wl, H=H)
    q, k, v = synth.make_qkv(wl, seed=seed, device=DEV)
    rows_np = synth.sample_rows(wl.L, wl.S, seed)
    rows = torch.from_numpy(rows_np).to(DEV)
    ref_mse, ref_label = svg.svg_profile_heads(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows)
    torch.cuda.synchronize()
    ref_mse, ref_label = ref_mse.cpu().double().numpy(), ref_label.cpu().numpy()
    gap = np.abs(ref_mse[..., 0] - ref_mse[..., 1]) / np.maximum(ref_mse.max(-1), 1e-300)
    bound = _bounds(q, k, v, wl, rows_np)
    if against_oracle:
        qn, kn, vn = (t.to("cpu", torch.float64).numpy() for t in (q, k, v))
        or_mse, or_label = oracle.profile_heads(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, rows_np)
        or_gap = np.abs(or_mse[..., 0] - or_mse[..., 1]) / np.maximum(or_mse.max(-1), 1e-300)
    for _ in range(2):  # two calls in a row share the static array
        mse = torch.full((wl.B, wl.H, 2), -1.0, dtype=torch.float32, device=DEV)
        label = torch.full((wl.B, wl.H), -1, dtype=torch.int8, device=DEV)
        st = _noalloc_raw(q, k, v, wl.N, wl.F, wl.a1, wl.a2, rows, mse, label)
        assert st == 0, svg.lib.svg_last_error().decode()
        torch.cuda.synchronize()
        got_mse, got_label = mse.cpu().double().numpy(), label.cpu().numpy()
        assert np.all(got_mse >= 0)
        # both calls are within the bound of the exact value, so within twice it of each other
        assert np.all(np.abs(got_mse - ref_mse) <= 2 * bound)
        decided = gap > 1e-3
        np.testing.assert_array_equal(got_label[decided], ref_label[decided])
        if against_oracle:
            assert np.all(np.abs(got_mse - or_mse) <= bound)
            np.testing.assert_array_equal(got_label[or_gap > 1e-3], or_label[or_gap > 1e-3])


def test_noalloc_matches_oracle_small():
    _check_against_workspace_version(synth.WORKLOADS["small"], seed=2, against_oracle=True)


def test_noalloc_matches_workspace_version_small():
    _check_against_workspace_version(synth.WORKLOADS["small"], seed=3)


def test_noalloc_matches_workspace_version_video_shape():
    # HunyuanVideo frame geometry with 8 heads: the default key split would
    # exceed the static array, so this exercises the re-chunked path.
    _check_against_workspace_version(synth.WORKLOADS["hunyuan"], seed=4, H=8)


def test_noalloc_rejects_shapes_beyond_the_array():
    wl = synth.WORKLOADS["hunyuan"]
    # 1024 heads of d=128 with S=128 need > 16 MiB even with one key chunk;
    # the call is refused before anything is enqueued.
    shape = svg.svg_shape(1, 1024, wl.N, wl.F, wl.d, svg.SVG_BF16, 0.0)
    p = ctypes.c_void_p(1 << 20)
    st = svg.lib.svg_profile_heads_noalloc(ctypes.byref(shape), p, p, p, 3, 281, p, 128, p, p, None)
    assert st == 5  # SVG_ERR_WORKSPACE
    assert b"static" in svg.lib.svg_last_error()
