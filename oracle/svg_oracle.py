"""Plain fp64 CPU oracle for spatial/temporal sparse 3D attention.

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
imports it, and it never imports the CUDA library or any of its helpers.

Everything here is written as directly as possible from the definitions on
the pages, with explicit boolean masks and a full softmax in float64.  There
is no tiling, fusion or reordering, so a reader can check each function
against the passage it cites.

Sources (cited by page title and section):
  [SVG-R]  "Sparse Video-Gen" author rebuttal (paperhub.cn):
           Weakness 1 answer (token indexing, Spatial Head, Temporal Head);
           the later Weakness 1 answer on online profiling (profiling runs at
           every step and layer, right before 3D full attention; heads are
           labelled -1 spatial / +1 temporal).
  [SVG-A]  "Sparse VideoGen: Accelerating Video Diffusion Transformers with
           Spatial-Temporal Sparsity" (newx.sg), Abstract and AI Summary
           (online profiling classifies heads; a hardware-efficient layout
           transformation; custom kernels).
  [SVG2]   SVG2 explainer (gist.science), section 2.A "Semantic-Aware
           Permutation" (a token permutation applied before attention and
           undone after it leaves the result mathematically unchanged).
  [SvDiT]  "Sparse-vDiT" review (pith.science), "What carries the argument"
           and "The reading": per-head modes {full, skip, diagonal,
           multi-diagonal, vertical stripe}; skipped heads have their output
           zeroed; the multi-diagonal pattern is turned into a diagonal one by
           a token rearrangement.

Readings taken where the pages are silent or garbled:
  * Temporal mask: the (i, j) form |j1 - j2| < a2 is authoritative.  The
    printed slash equivalence (with k ranging over 0 <= k < 2N-1) is garbled
    and would also admit wrap-around pairs; it is not used.
  * Softmax scale 1/sqrt(d) (textbook scaled dot-product attention).
  * Profiling: the caller passes the sampled query rows.  For each head,
    O_dense, O_spatial and O_temporal are the exact attention outputs of those
    rows (no mask, spatial mask, temporal mask).  mse_s and mse_t are the means
    over S*d elements of (O_s - O_dense)**2 and (O_t - O_dense)**2.  The head
    is temporal iff mse_t < mse_s (a tie counts as spatial).
  * Labels are int8 0 (spatial) / 1 (temporal), which stand for the pages'
    -1 / +1.
  * Layout transformation: token (i, j) moves from frame-major position
    x = i*F + j to token-major position x' = j*N + i.
  * Mixed modes (widths from the workload definition): diagonal of width 2W
    keeps |x1 - x2| <= W; multi-diagonal of stride F and width 2h keeps
    |j1 - j2| <= h (the (i, j) form, as for the temporal mask); vertical
    stripe keeps the first P keys; skip gives a zero output.
"""
from __future__ import annotations

import math

import numpy as np

SPATIAL = 0
TEMPORAL = 1


# --------------------------------------------------------------------------
# token indexing and masks  [SVG-R, Weakness 1 answer]
# --------------------------------------------------------------------------

def token_coords(N: int, F: int):
    """(i, j) of every flattened token x = i*F + j, 0 <= i < N, 0 <= j < F."""
    x = np.arange(N * F)
    return x // F, x % F


def spatial_mask(N: int, F: int, a1: int, rows=None) -> np.ndarray:
    """f_s[x1, x2] = 1 iff |i1 - i2| < a1  [SVG-R, Spatial Head].

    ``rows`` restricts the query side to the given flattened positions.
    """
    i, _ = token_coords(N, F)
    iq = i if rows is None else i[np.asarray(rows)]
    return np.abs(iq[:, None] - i[None, :]) < a1


def temporal_mask(N: int, F: int, a2: int, rows=None) -> np.ndarray:
    """f_t[x1, x2] = 1 iff |j1 - j2| < a2  [SVG-R, Temporal Head]."""
    _, j = token_coords(N, F)
    jq = j if rows is None else j[np.asarray(rows)]
    return np.abs(jq[:, None] - j[None, :]) < a2


def head_mask(label: int, N: int, F: int, a1: int, a2: int, rows=None) -> np.ndarray:
    """The mask a head of the given label uses, in the original layout."""
    if int(label) == TEMPORAL:
        return temporal_mask(N, F, a2, rows)
    return spatial_mask(N, F, a1, rows)


def banded_mask(L: int, G: int, a: int, rows=None) -> np.ndarray:
    """Block-banded mask over groups of G consecutive tokens:
    keep (x, y) iff |floor(x/G) - floor(y/G)| < a.

    [SVG-R, Spatial Head] states that the spatial mask is of this form with
    G = F, a = a1; the layout transformation [SVG-A] makes the temporal mask
    of this form with G = N, a = a2.
    """
    x = np.arange(L)
    g = x // G
    gq = g if rows is None else g[np.asarray(rows)]
    return np.abs(gq[:, None] - g[None, :]) < a


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def attention_probs(q, k, mask=None, scale=None) -> np.ndarray:
    """Row-wise softmax of scale * q k^T over the unmasked keys, in float64.

    q [R, d], k [L, d], mask [R, L] bool or None.  Masked entries get
    probability 0.  The row maximum is subtracted before exponentiating.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    if scale is None:
        scale = default_scale(q.shape[-1])
    s = (q @ k.T) * scale
    if mask is not None:
        s = np.where(mask, s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=-1, keepdims=True)


def attention(q, k, v, mask=None, scale=None) -> np.ndarray:
    """softmax(scale * q k^T + mask) v for one head, in float64."""
    p = attention_probs(q, k, mask, scale)
    return p @ np.asarray(v, dtype=np.float64)


def attention_rows(q, k, v, rows, mask_fn, scale=None, chunk=256) -> np.ndarray:
    """Attention of the query rows ``rows`` of one head.

    q, k, v [L, d]; ``mask_fn(rows_chunk)`` returns the [r, L] mask (or None
    for dense).  Rows are processed in chunks only to bound memory.
    """
    rows = np.asarray(rows)
    out = np.empty((rows.size, np.shape(v)[-1]), dtype=np.float64)
    for s0 in range(0, rows.size, chunk):
        rr = rows[s0:s0 + chunk]
        m = mask_fn(rr)
        out[s0:s0 + chunk] = attention(np.asarray(q)[rr], k, v, m, scale)
    return out


# --------------------------------------------------------------------------
# online profiling  [SVG-R, online-profiling answer; SVG-A, Abstract]
# --------------------------------------------------------------------------

def profile_heads(q, k, v, N: int, F: int, a1: int, a2: int, rows, scale=None):
    """Per-head spatial/temporal classification from sampled query rows.

    q, k, v: [B, H, L, d].  rows: [S] flattened query positions.
    Returns mse [B, H, 2] float64 (mse_s, mse_t) and label [B, H] int8.
    """
    q = np.asarray(q)
    B, H, L, d = q.shape
    rows = np.asarray(rows)
    ms = spatial_mask(N, F, a1, rows)
    mt = temporal_mask(N, F, a2, rows)
    mse = np.zeros((B, H, 2), dtype=np.float64)
    label = np.zeros((B, H), dtype=np.int8)
    for b in range(B):
        for h in range(H):
            qr = np.asarray(q[b, h], dtype=np.float64)[rows]
            kh = np.asarray(k[b, h], dtype=np.float64)
            vh = np.asarray(v[b, h], dtype=np.float64)
            o_dense = attention(qr, kh, vh, None, scale)
            o_s = attention(qr, kh, vh, ms, scale)
            o_t = attention(qr, kh, vh, mt, scale)
            mse[b, h, 0] = np.mean((o_s - o_dense) ** 2)
            mse[b, h, 1] = np.mean((o_t - o_dense) ** 2)
            label[b, h] = TEMPORAL if mse[b, h, 1] < mse[b, h, 0] else SPATIAL
    return mse, label


# --------------------------------------------------------------------------
# layout transformation  [SVG-A; SVG2 2.A]
# --------------------------------------------------------------------------

def token_major_index(N: int, F: int) -> np.ndarray:
    """pi[x] = j*N + i for x = i*F + j: the frame-major -> token-major map."""
    i, j = token_coords(N, F)
    return (j * N + i).astype(np.int64)


def permute(x, N: int, F: int) -> np.ndarray:
    """xp[..., pi[x], :] = x[..., x, :] along the token axis (axis -2)."""
    x = np.asarray(x)
    pi = token_major_index(N, F)
    out = np.empty_like(x)
    out[..., pi, :] = x
    return out


def unpermute(xp, N: int, F: int) -> np.ndarray:
    """Inverse of ``permute``: x[..., x, :] = xp[..., pi[x], :]."""
    xp = np.asarray(xp)
    pi = token_major_index(N, F)
    return xp[..., pi, :]


# --------------------------------------------------------------------------
# sparse attention output (ground truth for the whole call)
# --------------------------------------------------------------------------

def sparse_attention(q, k, v, label, N: int, F: int, a1: int, a2: int, scale=None,
                     rows=None) -> np.ndarray:
    """Each head's attention under its label's mask, in the ORIGINAL layout.

    q, k, v [B, H, L, d]; label [B, H].  With ``rows`` given, only those query
    rows are computed (returns [B, H, len(rows), d]).
    """
    q = np.asarray(q)
    B, H, L, d = q.shape
    R = L if rows is None else len(rows)
    out = np.zeros((B, H, R, d), dtype=np.float64)
    all_rows = np.arange(L) if rows is None else np.asarray(rows)
    for b in range(B):
        for h in range(H):
            lab = int(np.asarray(label)[b, h])
            out[b, h] = attention_rows(
                np.asarray(q[b, h], np.float64), np.asarray(k[b, h], np.float64),
                np.asarray(v[b, h], np.float64), all_rows,
                lambda rr, lab=lab: head_mask(lab, N, F, a1, a2, rr), scale)
    return out


def dense_attention(q, k, v, scale=None, rows=None) -> np.ndarray:
    """Unmasked attention of every head (optionally only ``rows``)."""
    q = np.asarray(q)
    B, H, L, d = q.shape
    all_rows = np.arange(L) if rows is None else np.asarray(rows)
    out = np.zeros((B, H, all_rows.size, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            out[b, h] = attention_rows(
                np.asarray(q[b, h], np.float64), np.asarray(k[b, h], np.float64),
                np.asarray(v[b, h], np.float64), all_rows, lambda rr: None, scale)
    return out


def sparse_attention_via_layout(q, k, v, label, N: int, F: int, a1: int, a2: int,
                                scale=None) -> np.ndarray:
    """The same result computed the way the method runs it: temporal heads are
    permuted to token-major order, attended under the block-banded mask with
    G = N, a = a2, and the output permuted back; spatial heads use the
    block-banded mask with G = F, a = a1 in place.  [SVG-A; SVG2 2.A]
    """
    q = np.asarray(q)
    B, H, L, d = q.shape
    out = np.zeros((B, H, L, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            if int(np.asarray(label)[b, h]) == TEMPORAL:
                qp, kp, vp = (permute(t[b, h], N, F) for t in (q, k, v))
                op = attention(qp, kp, vp, banded_mask(L, N, a2), scale)
                out[b, h] = unpermute(op, N, F)
            else:
                out[b, h] = attention(q[b, h], k[b, h], v[b, h], banded_mask(L, F, a1), scale)
    return out


# --------------------------------------------------------------------------
# block list (which key tiles a query tile touches)
# --------------------------------------------------------------------------

def block_list(mask: np.ndarray, Bq: int, Bk: int):
    """Brute-force tile classification of an explicit mask.

    Returns (active, full), each bool [ceil(Lq/Bq), ceil(Lk/Bk)]: a tile is
    active iff any of its elements is unmasked and full iff all are.  Tiles
    at the ragged edge cover only the rows/columns that exist.
    """
    Lq, Lk = mask.shape
    nq, nk = -(-Lq // Bq), -(-Lk // Bk)
    active = np.zeros((nq, nk), dtype=bool)
    full = np.zeros((nq, nk), dtype=bool)
    for qb in range(nq):
        for kb in range(nk):
            t = mask[qb * Bq:(qb + 1) * Bq, kb * Bk:(kb + 1) * Bk]
            active[qb, kb] = bool(t.any())
            full[qb, kb] = bool(t.all())
    return active, full


# --------------------------------------------------------------------------
# mixed sparse patterns  [SvDiT]
# --------------------------------------------------------------------------

MODE_FULL, MODE_SKIP, MODE_DIAGONAL, MODE_MULTIDIAG, MODE_STRIPE = 0, 1, 2, 3, 4


def window_mask(L: int, W: int, rows=None) -> np.ndarray:
    """Diagonal band: keep (x, y) iff |x - y| <= W."""
    x = np.arange(L)
    xq = x if rows is None else x[np.asarray(rows)]
    return np.abs(xq[:, None] - x[None, :]) <= W


def prefix_mask(L: int, P: int, rows=None) -> np.ndarray:
    """Vertical stripe: keep (x, y) iff y < P."""
    R = L if rows is None else len(rows)
    return np.broadcast_to(np.arange(L)[None, :] < P, (R, L)).copy()


def mode_mask(mode: int, N: int, F: int, window: int, md_half: int, stripe: int, rows=None):
    """The mask of one mixed-pattern head in the original layout (None for skip)."""
    L = N * F
    R = L if rows is None else len(rows)
    if mode == MODE_FULL:
        return np.ones((R, L), dtype=bool)
    if mode == MODE_DIAGONAL:
        return window_mask(L, window, rows)
    if mode == MODE_MULTIDIAG:
        return temporal_mask(N, F, md_half + 1, rows)  # |j1 - j2| <= md_half
    if mode == MODE_STRIPE:
        return prefix_mask(L, stripe, rows)
    if mode == MODE_SKIP:
        return None
    raise ValueError(mode)


def mixed_attention(q, k, v, modes, N: int, F: int, window: int, md_half: int, stripe: int, scale=None,
                    rows=None) -> np.ndarray:
    """Each head under its mode; skipped heads give zeros.  [B, H, R, d]."""
    q = np.asarray(q)
    B, H, L, d = q.shape
    all_rows = np.arange(L) if rows is None else np.asarray(rows)
    out = np.zeros((B, H, all_rows.size, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            m = int(np.asarray(modes)[b, h])
            if m == MODE_SKIP:
                continue
            out[b, h] = attention_rows(
                np.asarray(q[b, h], np.float64), np.asarray(k[b, h], np.float64),
                np.asarray(v[b, h], np.float64), all_rows,
                lambda rr, m=m: mode_mask(m, N, F, window, md_half, stripe, rr), scale)
    return out


# --------------------------------------------------------------------------
# offline mode search  [SvDiT: "What carries the argument"; referee report on
# Sec. 4.2, Eq. (2)]
# --------------------------------------------------------------------------

SEARCH_MODES = (MODE_SKIP, MODE_DIAGONAL, MODE_MULTIDIAG, MODE_STRIPE)


def mode_sparsity(mode: int, N: int, F: int, window: int, md_half: int, stripe: int) -> float:
    """Share of the L*L (query, key) pairs a mode does not compute, counted
    from its mask (one row at a time)."""
    L = N * F
    if mode == MODE_SKIP:
        return 1.0
    kept = 0
    for r0 in range(0, L, 512):
        rows = np.arange(r0, min(L, r0 + 512))
        kept += int(mode_mask(mode, N, F, window, md_half, stripe, rows).sum())
    return 1.0 - kept / float(L * L)


def mode_search(q, k, v, N: int, F: int, rows, window: int, md_half: int, stripe: int, lam: float = 0.5,
                eps: float = 1.0, scale=None, sparsity=None):
    """Per head and sparse mode i: L_i = MSE(O_i - O_dense) + lam * (1 - S_i)
    over the sampled rows; the head takes the smallest L_i unless all exceed
    eps (then full attention).  Returns loss [B, H, 4] (skip, diagonal,
    multi-diagonal, stripe) and mode [B, H].  Readings: Eq. (2)'s
    lam * (1 - S_i) (not the pseudocode's lam * S_i); eps compared with L_i;
    the MSE estimated on the sampled rows."""
    q = np.asarray(q)
    B, H, L, d = q.shape
    rows = np.asarray(rows)
    if sparsity is None:
        sparsity = [mode_sparsity(m, N, F, window, md_half, stripe) for m in SEARCH_MODES]
    loss = np.zeros((B, H, 4))
    mode = np.zeros((B, H), dtype=np.int8)
    for b in range(B):
        for h in range(H):
            qr = np.asarray(q[b, h], np.float64)[rows]
            kh, vh = np.asarray(k[b, h], np.float64), np.asarray(v[b, h], np.float64)
            o_dense = attention(qr, kh, vh, None, scale)
            for t, m in enumerate(SEARCH_MODES):
                if m == MODE_SKIP:
                    o_m = np.zeros_like(o_dense)
                else:
                    o_m = attention(qr, kh, vh, mode_mask(m, N, F, window, md_half, stripe, rows), scale)
                loss[b, h, t] = np.mean((o_m - o_dense) ** 2) + lam * (1.0 - sparsity[t])
            best = int(np.argmin(loss[b, h]))
            mode[b, h] = MODE_FULL if loss[b, h, best] > eps else SEARCH_MODES[best]
    return loss, mode
