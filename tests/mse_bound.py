"""Error bounds for the profiling MSEs, derived from the kernels' rounding.

The profiling kernels ("Sparse Video-Gen", the Weakness 1 answer on online
profiling) compute, per sampled row, the attention output with no mask (O)
and under a restricted mask B (O_B), and report mse = mean (O_B - O)^2.  The
GPU differs from the exact fp64 value in a few known places:

  * each softmax weight w_y = exp(s_y - m) is evaluated with relative error
    u_y: the bf16 rounding of the weight for the P V product (2^-8), the
    exponential itself (at most 1.02e-4 for the FMA-pipe cubic, about 2^-22
    for ex2.approx), and the fp32 score (products of bf16 values are exact;
    the fp32 sum over d terms and the fp32 scale-and-shift add a relative
    error of at most d 2^-24 sum|q_c k_c| scale + 2^-23 |x| in the exponent);
  * the three outputs of a row share the rounded weights, and each row sum
    adds up the same rounded weights its P V product sees, so O and O_B are
    exact convex combinations of V rows with perturbed weights; to first order
        |O_B^ - O_B - (O^ - O)| <= sum_y u_y |p^B_y [y in B] (v_y - O_B) - p_y (v_y - O)|
    (p the exact softmax weights over all keys, p^B those over B);
  * the fp32 accumulation of the P V products and of the row sums: at most
    n_add 2^-23 sum_y p_y |v_y| per output element, with n_add the number of
    fp32 additions into one accumulator (one per 16-key MMA step, plus the
    rescales and the chunk combine), and a final fp32 division.

With b the resulting per-element bound on the error of D = O_B - O,
    |mse_gpu - mse| <= mean over (rows, d) of (2 |D| b + b^2).
The bound scales with mse itself (the first-order term is proportional to D
where the band holds most of the mass), so it is a relative bar that a value
wrong by a few per cent fails.
"""
from __future__ import annotations

import numpy as np

U_BF16 = 2.0 ** -8       # relative rounding of a weight to bf16 (round to nearest)
U_EXP_BF16 = 1.1e-4      # exponentials of the tensor-core path (the cubic's 1.02e-4 bounds both kinds)
U_EXP_F32 = 2.0 ** -21   # ex2.approx on the fp32 CUDA-core path


def _row_terms(q, k, v, rows, scale, fp32_weights):
    """Exact weights and per-key relative error bounds of the sampled rows."""
    qr = q[rows]
    s = scale * (qr @ k.T)                                   # [S, L]
    m = s.max(1, keepdims=True)
    w = np.exp(s - m)
    d = q.shape[1]
    sabs = scale * (np.abs(qr) @ np.abs(k).T)
    x = (s - m) * np.log2(np.e)
    u = np.log(2.0) * (np.log2(np.e) * d * 2.0 ** -24 * sabs + 2.0 ** -23 * np.abs(x))
    u += U_EXP_F32 if fp32_weights else (U_BF16 + U_EXP_BF16)
    return w, u


def _variant_bound(w, u, v, keep, n_add):
    """Per-element bound [S, d] on the error of D = O_B - O, and D itself.
    keep: [S, L] bool mask of B, or None for the skip mode (O_B = 0).

    The first-order sum is evaluated with |v_y - c| <= |v_y| + |c| so that
    it needs only matrix products; for y in B, p^B_y = p_y / beta with
    beta = W_B / W, so that key's term is at most
        p_y ((1/beta - 1)(|v_y| + |O_B|) + |D|)."""
    W = w.sum(1, keepdims=True)
    p = w / W
    absv = np.abs(v)
    O = p @ v
    acc = n_add * 2.0 ** -23 * (p @ absv) + 2.0 ** -23 * np.abs(O)
    um = float(u.max())
    if keep is None:
        up = u * p
        first = up @ absv + np.abs(O) * up.sum(1, keepdims=True)
        second = 4.0 * um ** 2 * (p @ absv + np.abs(O))
        return first * (1 + 4 * um) + acc + second, -O
    wb = np.where(keep, w, 0.0)
    WB = wb.sum(1, keepdims=True)
    beta = WB / W
    pb = wb / np.where(WB > 0, WB, 1.0)
    OB = pb @ v
    D = OB - O
    upb = np.where(keep, u * p, 0.0)   # u_y p_y on B
    upo = u * p - upb                   # u_y p_y off B
    cB, cO = upb.sum(1, keepdims=True), upo.sum(1, keepdims=True)
    inv = np.where(beta > 0, 1.0 / np.where(beta > 0, beta, 1.0) - 1.0, 0.0)
    first = inv * (upb @ absv + np.abs(OB) * cB) + np.abs(D) * cB + (upo @ absv + np.abs(O) * cO)
    acc = acc + n_add * 2.0 ** -23 * (pb @ absv) + 2.0 ** -23 * np.abs(OB)
    second = 4.0 * um ** 2 * (pb @ absv + p @ absv + np.abs(OB) + np.abs(O))
    return first * (1 + 4 * um) + acc + second, D


def mse_error_bounds(q, k, v, rows, masks, scale=None, fp32_weights=False):
    """Bounds on |mse_gpu - mse_exact| for one head.

    q, k, v: [L, d] fp64 (the exact values the GPU was given).  rows: the
    sampled rows.  masks: list of [S, L] bool arrays (None = the skip mode).
    Returns (bounds, mse_exact) as arrays with one entry per mask."""
    q, k, v = (np.asarray(t, np.float64) for t in (q, k, v))
    rows = np.asarray(rows)
    L, d = k.shape
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    w, u = _row_terms(q, k, v, rows, scale, fp32_weights)
    # fp32 additions into one accumulator: one per key on the CUDA-core path;
    # one per 16-key MMA step, a rescale per 128-key tile and the chunk combine
    # on the tensor-core path
    n_add = L + 8 if fp32_weights else (L + 15) // 16 + 2 * ((L + 127) // 128) + 8
    bounds, exact = [], []
    for keep in masks:
        b, D = _variant_bound(w, u, v, keep, n_add)
        bounds.append(float(np.mean(2.0 * np.abs(D) * b + b * b)))
        exact.append(float(np.mean(D * D)))
    return np.array(bounds), np.array(exact)
