"""ctypes binding of libsvg.so, the CUDA library behind include/svg.h.

Argument marshalling only: every step of the computation runs in the
library's kernels.  PyTorch supplies device memory (outputs and workspaces
are allocated with torch when the caller does not pass them) and the current
CUDA stream.  Importing this module raises ImportError if libsvg.so has not
been built -- there is no fallback path.

Function names match the C entry points.  Tensors are contiguous CUDA
tensors (bf16 or fp32), [B, H, L, d] by default or [B, L, H, d] with
layout="blhd", with L = N * F in frame-major order (token (i, j) at row
i*F + j); labels are int8 [B, H] with 0 = spatial and 1 = temporal.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

# SVG_LIB names another build of the same library (the range-checked
# libsvg_debug.so in the tests); the default is the in-tree libsvg.so.
LIB_PATH = os.environ.get("SVG_LIB") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsvg.so")

SVG_OK = 0
SVG_BF16 = 0
SVG_FP32 = 1
SVG_TF32 = 2
SPATIAL = 0
TEMPORAL = 1
SVG_DEV_TIMEOUT = 0x1
SVG_DEV_RANGE = 0x2
SVG_DEV_BOUNDS = 0x4
SVG_LAYOUT_BHLD = 0
SVG_LAYOUT_BLHD = 1
LAYOUTS = {"bhld": SVG_LAYOUT_BHLD, "blhd": SVG_LAYOUT_BLHD}

# Every symbol include/svg.h declares.
EXPORTED = (
    "svg_abi_version", "svg_status_string", "svg_last_error", "svg_attn_tile", "svg_block_list",
    "svg_profile_workspace_size", "svg_workspace_size", "svg_profile_heads", "svg_permute", "svg_permute_qkv", "svg_unpermute",
    "svg_block_sparse_attn", "svg_banded_attn", "svg_dense_attn", "svg_sparse_3d_attn_workspace_size",
    "svg_sparse_3d_attn", "svg_profile_heads_noalloc", "svg_selftest_wait_bound", "svg_mixed_attn",
    "svg_mixed_3d_attn_workspace_size", "svg_mixed_3d_attn", "svg_sparse_3d_attn_host_workspace_size",
    "svg_sparse_3d_attn_host", "svg_mode_search_workspace_size", "svg_mode_search", "svg_block_sparse_attn_fused",
    "svg_mixed_attn_fused", "svg_sparse_3d_attn_plan", "svg_semantic_attn_workspace_size", "svg_semantic_attn",
    "svg_kmeans_workspace_size", "svg_kmeans", "svg_semantic_3d_attn_workspace_size", "svg_semantic_3d_attn",
    "svg_head_shard", "svg_sparse_3d_attn_shard_workspace_size", "svg_sparse_3d_attn_shard", "svg_debug_checks",
)

MODE_FULL, MODE_SKIP, MODE_DIAGONAL, MODE_MULTIDIAG, MODE_STRIPE = 0, 1, 2, 3, 4


class SvgError(RuntimeError):
    """A libsvg entry point returned a non-OK status."""

    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class svg_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("F", ctypes.c_int32),
                ("d", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float),
                ("layout", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_Z = ctypes.c_size_t


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m sparse_attention_video_profile_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "svg_abi_version": (_I, []),
        "svg_debug_checks": (_I, []),
        "svg_status_string": (ctypes.c_char_p, [_I]),
        "svg_last_error": (ctypes.c_char_p, []),
        "svg_attn_tile": (_I, [_I, _I, _P, _P]),
        "svg_block_list": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P]),
        "svg_profile_workspace_size": (_Z, [_P, _I]),
        "svg_workspace_size": (_Z, [_P, _I]),
        "svg_profile_heads": (_I, [_P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _Z, _P]),
        "svg_permute": (_I, [_P, _P, _P, _P, _P]),
        "svg_permute_qkv": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "svg_unpermute": (_I, [_P, _P, _P, _P, _P]),
        "svg_block_sparse_attn": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P]),
        "svg_banded_attn": (_I, [_P, _P, _P, _P, _P, _I, _I, _P, _P]),
        "svg_dense_attn": (_I, [_P, _P, _P, _P, _P, _P, _P]),
        "svg_sparse_3d_attn_workspace_size": (_Z, [_P, _I, _I]),
        "svg_sparse_3d_attn": (_I, [_P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _Z, _P, _P]),
        "svg_profile_heads_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P]),
        "svg_selftest_wait_bound": (_I, [_P, _P, _P, _P, _P, ctypes.c_uint64, _P, _P]),
        "svg_mixed_attn": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
        "svg_mixed_3d_attn_workspace_size": (_Z, [_P]),
        "svg_mixed_3d_attn": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _Z, _P, _P]),
        "svg_sparse_3d_attn_host_workspace_size": (_Z, [_P, _I, _I, _I]),
        "svg_sparse_3d_attn_host": (_I, [_P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _I, _P, _Z, _P, _P]),
        "svg_mode_search_workspace_size": (_Z, [_P, _I]),
        "svg_block_sparse_attn_fused": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _P, _P]),
        "svg_mixed_attn_fused": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
        "svg_sparse_3d_attn_plan": (_I, [_P, _I, _P, _P, _P]),
        "svg_semantic_attn_workspace_size": (_Z, [_P, _I, _I]),
        "svg_semantic_attn": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, ctypes.c_float, _P, _P, _Z, _P, _P]),
        "svg_kmeans_workspace_size": (_Z, [_P, _I]),
        "svg_kmeans": (_I, [_P, _P, _I, _I, _P, _P, _P, _Z, _P, _P]),
        "svg_semantic_3d_attn_workspace_size": (_Z, [_P, _I, _I]),
        "svg_semantic_3d_attn": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, ctypes.c_float, _P, _P, _P, _P, _Z, _P, _P]),
        "svg_mode_search": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_float, ctypes.c_float, _P, _P, _P, _Z,
                                 _P]),
        "svg_head_shard": (_I, [_I, _I, _I, _P, _P]),
        "svg_sparse_3d_attn_shard_workspace_size": (_Z, [_P, _I, _I, _I, _I]),
        "svg_sparse_3d_attn_shard": (_I, [_P, _I, _I, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _Z, _P, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _check(status: int) -> None:
    if status != SVG_OK:
        name = lib.svg_status_string(status).decode()
        msg = lib.svg_last_error().decode()
        raise SvgError(status, f"{name}: {msg}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SVG_BF16
    if t.dtype == torch.float32:
        return SVG_FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def make_shape(x: torch.Tensor, N: int, F: int, scale: float = 0.0, layout: str = "bhld",
               tf32: bool = False) -> svg_shape:
    """The svg_shape of a q/k/v tensor: [B, H, L, d] (layout "bhld") or
    [B, L, H, d] ("blhd").  tf32=True (float32 tensors only) runs attention
    on the tensor cores in tf32 (SVG_TF32) instead of fp32 on the CUDA cores."""
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(LAYOUTS)}, got {layout!r}")
    if x.dim() != 4:
        raise ValueError(f"expected a [B, H, L, d] or [B, L, H, d] tensor, got {x.dim()} dims")
    if layout == "bhld":
        B, H, L, d = x.shape
    else:
        B, L, H, d = x.shape
    if L != N * F:
        raise ValueError(f"L = {L} but N*F = {N * F}")
    code = _dtype_code(x)
    if tf32:
        if code != SVG_FP32:
            raise TypeError("tf32=True takes float32 tensors")
        code = SVG_TF32
    return svg_shape(B, H, N, F, d, code, float(scale), LAYOUTS[layout])


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _same(ref: torch.Tensor, *ts: torch.Tensor):
    for t in ts:
        if t.shape != ref.shape or t.dtype != ref.dtype or t.device != ref.device:
            raise ValueError("q, k, v (and outputs) must share shape, dtype and device")


# ------------------------------------------------------------------ host-only

def svg_abi_version() -> int:
    return int(lib.svg_abi_version())


def svg_attn_tile(dtype: int, d: int):
    bq, bk = ctypes.c_int32(), ctypes.c_int32()
    _check(lib.svg_attn_tile(dtype, d, ctypes.byref(bq), ctypes.byref(bk)))
    return bq.value, bk.value


def svg_block_list(L: int, G: int, a: int, Bq: int, Bk: int):
    """(kb_lo, kb_hi, full_lo, full_hi) int32 numpy arrays, one entry per query tile."""
    nq = -(-L // Bq)
    arrs = [np.zeros(nq, dtype=np.int32) for _ in range(4)]
    _check(lib.svg_block_list(L, G, a, Bq, Bk, *(a_.ctypes.data_as(ctypes.c_void_p) for a_ in arrs)))
    return tuple(arrs)


def svg_profile_workspace_size(shape: svg_shape, S: int) -> int:
    return int(lib.svg_profile_workspace_size(ctypes.byref(shape), S))


def svg_workspace_size(shape: svg_shape, n_temporal_heads_max: int) -> int:
    """Workspace of the step-by-step call: [profiling | qp | kp | vp | op]."""
    return int(lib.svg_workspace_size(ctypes.byref(shape), n_temporal_heads_max))


def svg_sparse_3d_attn_plan(shape: svg_shape, a2: int):
    """(separate_tiles, fused_tiles, fused): the whole call's layout choice."""
    sep, fz, fu = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
    _check(lib.svg_sparse_3d_attn_plan(ctypes.byref(shape), a2, ctypes.byref(sep), ctypes.byref(fz), ctypes.byref(fu)))
    return int(sep.value), int(fz.value), bool(fu.value)


def svg_sparse_3d_attn_workspace_size(shape: svg_shape, a2: int, S: int) -> int:
    return int(lib.svg_sparse_3d_attn_workspace_size(ctypes.byref(shape), a2, S))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ device calls

def svg_profile_heads(q, k, v, N: int, F: int, a1: int, a2: int, rows: torch.Tensor, *, mse=None, label=None,
                      workspace=None, scale: float = 0.0, layout: str = "bhld", stream=None):
    """Online profiling.  Returns (mse [B,H,2] f32, label [B,H] int8) on q's device."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout)
    if rows.dtype != torch.int32 or rows.device != q.device:
        raise ValueError("rows must be an int32 tensor on q's device")
    S = rows.numel()
    if mse is None:
        mse = torch.empty(shape.B, shape.H, 2, dtype=torch.float32, device=q.device)
    if label is None:
        label = torch.empty(shape.B, shape.H, dtype=torch.int8, device=q.device)
    need = svg_profile_workspace_size(shape, S)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    _check(lib.svg_profile_heads(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), a1, a2, _ptr(rows), S, _ptr(mse),
                                 _ptr(label), _ptr(workspace), workspace.numel(), _stream(stream)))
    return mse, label


def svg_profile_heads_noalloc(q, k, v, N: int, F: int, a1: int, a2: int, rows: torch.Tensor, *, mse=None,
                              label=None, scale: float = 0.0, layout: str = "bhld", stream=None):
    """Online profiling without a workspace, for callers that cannot allocate
    device memory.  The library's fixed scratch array stands in for the
    workspace (see include/svg.h).  mse and label should be passed in by
    such callers; they are allocated here only for convenience."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout)
    if rows.dtype != torch.int32 or rows.device != q.device:
        raise ValueError("rows must be an int32 tensor on q's device")
    if mse is None:
        mse = torch.empty(shape.B, shape.H, 2, dtype=torch.float32, device=q.device)
    if label is None:
        label = torch.empty(shape.B, shape.H, dtype=torch.int8, device=q.device)
    _check(lib.svg_profile_heads_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), a1, a2, _ptr(rows),
                                         rows.numel(), _ptr(mse), _ptr(label), _stream(stream)))
    return mse, label


def svg_permute(x, N: int, F: int, label=None, *, out=None, layout: str = "bhld", stream=None):
    shape = make_shape(x, N, F, 0.0, layout)
    if out is None:
        out = torch.empty_like(x)
    _check(lib.svg_permute(ctypes.byref(shape), _ptr(x), _ptr(out), _ptr(label), _stream(stream)))
    return out


def svg_permute_qkv(q, k, v, N: int, F: int, label=None, *, out: Optional[Sequence] = None, layout: str = "bhld",
                    stream=None):
    _same(q, k, v)
    shape = make_shape(q, N, F, 0.0, layout)
    qp, kp, vp = out if out is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    _check(lib.svg_permute_qkv(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(qp), _ptr(kp), _ptr(vp),
                               _ptr(label), _stream(stream)))
    return qp, kp, vp


def svg_unpermute(xp, N: int, F: int, label=None, *, out=None, layout: str = "bhld", stream=None):
    shape = make_shape(xp, N, F, 0.0, layout)
    if out is None:
        out = torch.empty_like(xp)
    _check(lib.svg_unpermute(ctypes.byref(shape), _ptr(xp), _ptr(out), _ptr(label), _stream(stream)))
    return out


def svg_block_sparse_attn(q, k, v, qp, kp, vp, label, N: int, F: int, a1: int, a2: int, *, o=None, op=None,
                          status=None, scale: float = 0.0, layout: str = "bhld", tf32: bool = False, stream=None):
    """Returns (o, op): spatial heads' output in o, temporal heads' in op."""
    _same(q, k, v, qp, kp, vp)
    shape = make_shape(q, N, F, scale, layout, tf32=tf32)
    if o is None:
        o = torch.empty_like(q)
    if op is None:
        op = torch.empty_like(q)
    _check(lib.svg_block_sparse_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(qp), _ptr(kp), _ptr(vp),
                                     _ptr(o), _ptr(op), _ptr(label), a1, a2, _ptr(status), _stream(stream)))
    return o, op


def svg_block_sparse_attn_fused(q, k, v, label, N: int, F: int, a1: int, a2: int, *, o=None, status=None,
                                scale: float = 0.0, layout: str = "bhld", stream=None):
    """Block-sparse attention with the layout transformation fused in: every
    head's output lands frame-major in o (no permuted copies).  bf16."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout)
    if o is None:
        o = torch.empty_like(q)
    _check(lib.svg_block_sparse_attn_fused(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(label), a1,
                                           a2, _ptr(status), _stream(stream)))
    return o


def svg_banded_attn(q, k, v, N: int, F: int, G: int, a: int, *, o=None, status=None, scale: float = 0.0,
                    layout: str = "bhld", tf32: bool = False, stream=None):
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout, tf32=tf32)
    if o is None:
        o = torch.empty_like(q)
    _check(lib.svg_banded_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), G, a, _ptr(status),
                               _stream(stream)))
    return o


def svg_dense_attn(q, k, v, N: int, F: int, *, o=None, status=None, scale: float = 0.0, layout: str = "bhld",
                   tf32: bool = False, stream=None):
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout, tf32=tf32)
    if o is None:
        o = torch.empty_like(q)
    _check(lib.svg_dense_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(status),
                              _stream(stream)))
    return o


def svg_sparse_3d_attn(q, k, v, N: int, F: int, a1: int, a2: int, rows: torch.Tensor, *, o=None, mse=None,
                       label=None, workspace=None, status=None, scale: float = 0.0, layout: str = "bhld",
                       tf32: bool = False, stream=None):
    """One whole sparse 3D-attention call.  Returns (o, mse, label)."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout, tf32=tf32)
    S = rows.numel()
    if o is None:
        o = torch.empty_like(q)
    if mse is None:
        mse = torch.empty(shape.B, shape.H, 2, dtype=torch.float32, device=q.device)
    if label is None:
        label = torch.empty(shape.B, shape.H, dtype=torch.int8, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(svg_sparse_3d_attn_workspace_size(shape, a2, S), q.device)
    _check(lib.svg_sparse_3d_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), a1, a2, _ptr(rows), S,
                                  _ptr(mse), _ptr(label), _ptr(workspace), workspace.numel(), _ptr(status),
                                  _stream(stream)))
    return o, mse, label


def svg_head_shard(n_heads: int, rank: int, world: int):
    """(first, count): rank's contiguous block of the heads numbered over (b, h)."""
    first, count = ctypes.c_int32(), ctypes.c_int32()
    _check(lib.svg_head_shard(n_heads, rank, world, ctypes.byref(first), ctypes.byref(count)))
    return int(first.value), int(count.value)


def gather_heads(x: torch.Tensor, n_heads: int, rank: int, world: int, group=None) -> torch.Tensor:
    """Fills every rank's block of heads of x (shape [B, H, ...], this rank's
    block already written) from the other ranks, in place: one all-gather of
    blocks padded to the largest block.  Works on any torch.distributed
    backend (NCCL for device tensors, gloo for host tensors)."""
    import torch.distributed as dist
    flat = x.view(n_heads, -1)
    first, count = svg_head_shard(n_heads, rank, world)
    width = -(-n_heads // world)
    buf = torch.zeros(width, flat.shape[1], dtype=x.dtype, device=x.device)
    buf[:count] = flat[first:first + count]
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf, group=group)
    for r in range(world):
        f, c = svg_head_shard(n_heads, r, world)
        if r != rank and c:
            flat[f:f + c] = parts[r][:c]
    return x


def gather_output(o: torch.Tensor, n_heads: int, rank: int, world: int, layout: str = "bhld",
                  group=None) -> torch.Tensor:
    """gather_heads for an attention output in either layout.  In
    [B, L, H, d] a block of heads is not contiguous, so the blocks travel as
    a [B, H, L, d] copy that is written back afterwards."""
    if layout == "bhld":
        return gather_heads(o, n_heads, rank, world, group)
    if layout != "blhd":
        raise ValueError(f"layout must be one of {sorted(LAYOUTS)}, got {layout!r}")
    oh = o.transpose(1, 2).contiguous()
    gather_heads(oh, n_heads, rank, world, group)
    o.copy_(oh.transpose(1, 2))
    return o


def svg_sparse_3d_attn_shard(q, k, v, N: int, F: int, a1: int, a2: int, rows: torch.Tensor, rank: int, world: int, *,
                             o=None, mse=None, label=None, workspace=None, status=None, scale: float = 0.0,
                             layout: str = "bhld", tf32: bool = False, stream=None, gather: bool = False, group=None):
    """This rank's block of heads of one whole call (q, k, v are the full
    tensors).  Returns (o, mse, label) full-size; only this rank's heads are
    written unless gather=True, which then fills the rest from the other
    ranks (torch.distributed must be initialised)."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout, tf32=tf32)
    S = rows.numel()
    if o is None:
        o = torch.empty_like(q)
    if mse is None:
        mse = torch.empty(shape.B, shape.H, 2, dtype=torch.float32, device=q.device)
    if label is None:
        label = torch.empty(shape.B, shape.H, dtype=torch.int8, device=q.device)
    if workspace is None:
        need = int(lib.svg_sparse_3d_attn_shard_workspace_size(ctypes.byref(shape), rank, world, a2, S))
        workspace = alloc_workspace(need, q.device)
    _check(lib.svg_sparse_3d_attn_shard(ctypes.byref(shape), rank, world, _ptr(q), _ptr(k), _ptr(v), _ptr(o), a1, a2,
                                        _ptr(rows), S, _ptr(mse), _ptr(label), _ptr(workspace), workspace.numel(),
                                        _ptr(status), _stream(stream)))
    if gather and world > 1:
        n = shape.B * shape.H
        for t in (mse, label):
            gather_heads(t, n, rank, world, group)
        gather_output(o, n, rank, world, layout, group)
    return o, mse, label


def svg_mixed_attn_fused(q, k, v, mode, N: int, F: int, window: int, md_half: int, stripe: int, *, o=None,
                         status=None, scale: float = 0.0, layout: str = "bhld", stream=None):
    """Mixed-pattern attention with the multi-diagonal heads' layout fused in."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout)
    if o is None:
        o = torch.empty_like(q)
    _check(lib.svg_mixed_attn_fused(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(mode), window,
                                    md_half, stripe, _ptr(status), _stream(stream)))
    return o


def svg_mixed_attn(q, k, v, qp, kp, vp, mode, N: int, F: int, window: int, md_half: int, stripe: int, *,
                   o=None, op=None, status=None, scale: float = 0.0, layout: str = "bhld", stream=None):
    """Every head under its own mode (SVG_MODE_*), one launch.  Returns (o, op)."""
    _same(q, k, v, qp, kp, vp)
    shape = make_shape(q, N, F, scale, layout)
    if o is None:
        o = torch.empty_like(q)
    if op is None:
        op = torch.empty_like(q)
    _check(lib.svg_mixed_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(qp), _ptr(kp), _ptr(vp),
                              _ptr(o), _ptr(op), _ptr(mode), window, md_half, stripe, _ptr(status),
                              _stream(stream)))
    return o, op


def svg_mixed_3d_attn(q, k, v, mode, N: int, F: int, window: int, md_half: int, stripe: int, *, o=None,
                      workspace=None, status=None, scale: float = 0.0, layout: str = "bhld", stream=None):
    """One mixed-pattern call (permutation of multi-diagonal heads included)."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(int(lib.svg_mixed_3d_attn_workspace_size(ctypes.byref(shape))), q.device)
    _check(lib.svg_mixed_3d_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(mode), window,
                                 md_half, stripe, _ptr(workspace), workspace.numel(), _ptr(status),
                                 _stream(stream)))
    return o


def svg_sparse_3d_attn_host(q, k, v, N: int, F: int, a1: int, a2: int, rows, *, o=None, mse=None, label=None,
                            heads_per_chunk: int = 4, workspace=None, status=None, scale: float = 0.0,
                            device=None, tf32: bool = False, stream=None):
    """svg_sparse_3d_attn on host (CPU) tensors, copies overlapped with the
    kernels.  q, k, v (and o) should be pinned.  Returns (o, mse, label) as
    host tensors, valid after `stream` (the current stream) synchronises."""
    for t in (q, k, v):
        if t.device.type != "cpu":
            raise ValueError("svg_sparse_3d_attn_host takes host tensors")
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, tf32=tf32)
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    rows = rows.to(torch.int32).contiguous()
    if o is None:
        o = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if mse is None:
        mse = torch.empty(shape.B, shape.H, 2, dtype=torch.float32, pin_memory=True)
    if label is None:
        label = torch.empty(shape.B, shape.H, dtype=torch.int8, pin_memory=True)
    if workspace is None:
        need = int(lib.svg_sparse_3d_attn_host_workspace_size(ctypes.byref(shape), a2, rows.numel(), heads_per_chunk))
        workspace = alloc_workspace(need, dev)
    _check(lib.svg_sparse_3d_attn_host(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), a1, a2, _ptr(rows),
                                       rows.numel(), _ptr(mse), _ptr(label), heads_per_chunk, _ptr(workspace),
                                       workspace.numel(), _ptr(status), _stream(stream)))
    return o, mse, label


def svg_mode_search(q, k, v, N: int, F: int, rows, window: int, md_half: int, stripe: int, *, lam: float = 0.5,
                    epsilon: float = 1.0, loss=None, mode=None, workspace=None, scale: float = 0.0,
                    layout: str = "bhld", stream=None):
    """Sparse-vDiT mode selection per head.  Returns (loss [B,H,4]: skip,
    diagonal, multi-diagonal, stripe; mode [B,H] int8 SVG_MODE_*)."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout)
    if loss is None:
        loss = torch.empty(shape.B, shape.H, 4, dtype=torch.float32, device=q.device)
    if mode is None:
        mode = torch.empty(shape.B, shape.H, dtype=torch.int8, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(int(lib.svg_mode_search_workspace_size(ctypes.byref(shape), rows.numel())),
                                    q.device)
    _check(lib.svg_mode_search(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(rows), rows.numel(), window,
                               md_half, stripe, float(lam), float(epsilon), _ptr(loss), _ptr(mode), _ptr(workspace),
                               workspace.numel(), _stream(stream)))
    return loss, mode


def svg_semantic_attn(q, k, v, N: int, F: int, assign_q, assign_k, Cq: int, Ck: int, p: float, *, o=None,
                      selected=None, workspace=None, status=None, scale: float = 0.0, layout: str = "bhld",
                      stream=None):
    """SVG2-style attention given the token clusters (int32 [B,H,L] each).
    Returns (o, selected [B,H,Cq,ceil(Ck/32)] uint32 bitmask as int32)."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout)
    if o is None:
        o = torch.empty_like(q)
    if selected is None:
        selected = torch.empty(shape.B, shape.H, Cq, (Ck + 31) // 32, dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(int(lib.svg_semantic_attn_workspace_size(ctypes.byref(shape), Cq, Ck)), q.device)
    _check(lib.svg_semantic_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(assign_q),
                                 _ptr(assign_k), Cq, Ck, float(p), _ptr(selected), _ptr(workspace), workspace.numel(),
                                 _ptr(status), _stream(stream)))
    return o, selected


def svg_kmeans(x, N: int, F: int, C: int, iters: int, *, assign=None, centroids=None, workspace=None, status=None,
               layout: str = "bhld", stream=None):
    """k-means of every head's rows.  Returns (assign int32 [B,H,L], centroids float32 [B,H,C,d])."""
    shape = make_shape(x, N, F, 0.0, layout)
    if assign is None:
        assign = torch.empty(shape.B, shape.H, N * F, dtype=torch.int32, device=x.device)
    if centroids is None:
        centroids = torch.empty(shape.B, shape.H, C, shape.d, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = alloc_workspace(int(lib.svg_kmeans_workspace_size(ctypes.byref(shape), C)), x.device)
    _check(lib.svg_kmeans(ctypes.byref(shape), _ptr(x), C, iters, _ptr(assign), _ptr(centroids), _ptr(workspace),
                          workspace.numel(), _ptr(status), _stream(stream)))
    return assign, centroids


def svg_semantic_3d_attn(q, k, v, N: int, F: int, Cq: int, Ck: int, iters: int, p: float, *, o=None, assign_q=None,
                         assign_k=None, selected=None, workspace=None, status=None, scale: float = 0.0,
                         layout: str = "bhld", stream=None):
    """The whole SVG2-style call (k-means of Q and K, top-p, attention).
    Returns (o, assign_q, assign_k, selected)."""
    _same(q, k, v)
    shape = make_shape(q, N, F, scale, layout)
    L = N * F
    if o is None:
        o = torch.empty_like(q)
    if assign_q is None:
        assign_q = torch.empty(shape.B, shape.H, L, dtype=torch.int32, device=q.device)
    if assign_k is None:
        assign_k = torch.empty(shape.B, shape.H, L, dtype=torch.int32, device=q.device)
    if selected is None:
        selected = torch.empty(shape.B, shape.H, Cq, (Ck + 31) // 32, dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(int(lib.svg_semantic_3d_attn_workspace_size(ctypes.byref(shape), Cq, Ck)),
                                    q.device)
    _check(lib.svg_semantic_3d_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), Cq, Ck, iters, float(p),
                                    _ptr(assign_q), _ptr(assign_k), _ptr(selected), _ptr(workspace),
                                    workspace.numel(), _ptr(status), _stream(stream)))
    return o, assign_q, assign_k, selected


def selected_bits(selected, Ck: int):
    """[B,H,Cq,W] bitmask words -> [B,H,Cq,Ck] bool (host numpy)."""
    import numpy as np
    w = selected.cpu().numpy().astype(np.uint32)
    bits = (w[..., None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(*w.shape[:-1], -1)[..., :Ck].astype(bool)


def svg_selftest_wait_bound(q, k, v, N: int, F: int, status, *, wait_ns: int = 50_000_000, o=None,
                            layout: str = "bhld", stream=None):
    """Failure-detection self-test: the attention kernel with its loads
    withheld must time out, set SVG_DEV_TIMEOUT in `status` and exit."""
    shape = make_shape(q, N, F, 0.0, layout)
    if o is None:
        o = torch.empty_like(q)
    _check(lib.svg_selftest_wait_bound(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), int(wait_ns),
                                       _ptr(status), _stream(stream)))
    return o


class SparseAttention3D:
    """A reusable sparse 3D-attention call for one video shape: keeps its
    workspace between calls (svg_sparse_3d_attn: profiling, then attention
    with the layout transformation fused in or as separate passes)."""

    def __init__(self, N: int, F: int, a1: int, a2: int, scale: float = 0.0, layout: str = "bhld",
                 tf32: bool = False):
        self.N, self.F, self.a1, self.a2, self.scale, self.layout, self.tf32 = N, F, a1, a2, scale, layout, tf32
        self._ws = None

    def __call__(self, q, k, v, rows, *, o=None, mse=None, label=None, status=None, stream=None):
        shape = make_shape(q, self.N, self.F, self.scale, self.layout, self.tf32)
        need = svg_sparse_3d_attn_workspace_size(shape, self.a2, rows.numel())
        if self._ws is None or self._ws.numel() < need or self._ws.device != q.device:
            self._ws = alloc_workspace(need, q.device)
        return svg_sparse_3d_attn(q, k, v, self.N, self.F, self.a1, self.a2, rows, o=o, mse=mse, label=label,
                                  workspace=self._ws, status=status, scale=self.scale, layout=self.layout,
                                  tf32=self.tf32, stream=stream)
