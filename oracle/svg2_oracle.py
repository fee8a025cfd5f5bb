"""Plain fp64 CPU oracle for SVG2-style semantic-aware sparse attention.

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
imports it, and it never imports the CUDA library or any of its helpers.

Source: the SVG2 explainer (gist.science), section 2 "Methodology":
  2.A "Semantic-Aware Permutation" -- Q and K are clustered independently by
      k-means into C_q and C_k clusters; tokens are reordered so that each
      cluster is contiguous; the permutation is undone on the output, so the
      result equals attention over the same key sets in the original order.
  2.B "Centroid-Based Top-p Selection" -- attention scores are estimated
      between cluster centroids; for each query cluster the key clusters are
      sorted by estimated score and taken in that order until the cumulative
      score reaches p.
  2.C "Customized Attention Kernel" -- contiguous query clusters attend to
      the selected (variable-size) key clusters.

Readings taken where the page is silent:
  * k-means is Lloyd's algorithm with Euclidean distance, run for a fixed
    number of iterations from a deterministic start: centroid c is the row
    floor(c * L / C).  A row goes to its nearest centroid (ties: the lowest
    cluster index); a cluster's new centroid is the mean of its rows; an
    empty cluster keeps its centroid.
  * The permutation is stable: clusters in index order, rows of a cluster in
    their original order.
  * The centroid score of key cluster c_k for query cluster c_q is the
    attention mass the key cluster would get if all its n_k keys sat at its
    centroid: w = n_k * exp(scale * mu_q . mu_k), normalised over c_k.
    Clusters are sorted by w (ties: the lower index first) and the shortest
    prefix whose cumulative w reaches p is kept.  Empty key clusters have
    w = 0 and are never kept.
  * A query row attends to every key in the key clusters its query cluster
    keeps, and to no other key.
"""
from __future__ import annotations

import numpy as np


def _scale(d: int, scale):
    return (1.0 / np.sqrt(d)) if scale is None else float(scale)


def kmeans(x, C: int, iters: int):
    """Lloyd's algorithm on the rows of x [L, d] (fp64) from the rows
    floor(c L / C).  Returns (assign [L] int, centroids [C, d], counts [C])
    after `iters` assignment + update rounds; the returned assignment is the
    last round's, the centroids are the means of that assignment."""
    x = np.asarray(x, np.float64)
    L = x.shape[0]
    init = (np.arange(C) * L) // C
    mu = x[init].copy()
    assign = np.zeros(L, dtype=np.int64)
    counts = np.zeros(C, dtype=np.int64)
    for _ in range(iters):
        assign = nearest_centroid(x, mu)
        counts = np.bincount(assign, minlength=C)
        sums = np.zeros_like(mu)
        np.add.at(sums, assign, x)
        nz = counts > 0
        mu[nz] = sums[nz] / counts[nz, None]
    return assign, mu, counts


def nearest_centroid(x, mu):
    """Index of the nearest centroid (squared Euclidean distance) of every
    row; ties go to the lowest index (argmin returns the first)."""
    x = np.asarray(x, np.float64)
    mu = np.asarray(mu, np.float64)
    d2 = (x * x).sum(1)[:, None] - 2.0 * x @ mu.T + (mu * mu).sum(1)[None, :]
    return np.argmin(d2, axis=1)


def kmeans_objective(x, mu, assign) -> float:
    """Sum of squared distances of the rows to their assigned centroids."""
    x = np.asarray(x, np.float64)
    return float(((x - np.asarray(mu, np.float64)[np.asarray(assign)]) ** 2).sum())


def cluster_permutation(assign, C: int):
    """Stable order of the rows by cluster.  Returns (perm, offsets): the
    row at permuted position r is perm[r]; cluster c occupies permuted
    positions [offsets[c], offsets[c + 1])."""
    assign = np.asarray(assign)
    perm = np.argsort(assign, kind="stable")
    offsets = np.zeros(C + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(np.bincount(assign, minlength=C))
    return perm, offsets


def centroid_topp(mu_q, mu_k, n_k, p: float, scale=None):
    """Selected key clusters per query cluster: [C_q, C_k] bool."""
    mu_q = np.asarray(mu_q, np.float64)
    mu_k = np.asarray(mu_k, np.float64)
    n_k = np.asarray(n_k, np.float64)
    s = _scale(mu_q.shape[1], scale)
    logits = s * (mu_q @ mu_k.T)
    w = np.where(n_k[None, :] > 0, n_k[None, :] * np.exp(logits - logits.max(1, keepdims=True)), 0.0)
    w = w / w.sum(1, keepdims=True)
    Cq, Ck = w.shape
    sel = np.zeros((Cq, Ck), dtype=bool)
    for c in range(Cq):
        order = sorted(range(Ck), key=lambda j: (-w[c, j], j))
        acc = 0.0
        for j in order:
            if w[c, j] <= 0.0:
                break
            sel[c, j] = True
            acc += w[c, j]
            if acc >= p:
                break
    return sel


def svg2_mask(assign_q, assign_k, selected, rows=None):
    """mask[x, y] = True iff the query cluster of row x keeps the key cluster
    of key y (original token order)."""
    aq = np.asarray(assign_q)
    if rows is not None:
        aq = aq[np.asarray(rows)]
    return np.asarray(selected)[aq][:, np.asarray(assign_k)]


def svg2_attention_given(q, k, v, assign_q, assign_k, selected, scale=None, rows=None):
    """Attention of one head [L, d] (or of the query rows `rows`) under the
    cluster-pair mask, in the original order.  A row whose cluster keeps no
    key gets zeros."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    rr = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    s = _scale(q.shape[1], scale)
    out = np.zeros((rr.size, v.shape[1]))
    for c0 in range(0, rr.size, 256):
        r = rr[c0:c0 + 256]
        m = svg2_mask(assign_q, assign_k, selected, r)
        logits = np.where(m, s * (q[r] @ k.T), -np.inf)
        mx = logits.max(1, keepdims=True)
        ok = np.isfinite(mx[:, 0])
        e = np.zeros_like(logits)
        e[ok] = np.exp(logits[ok] - mx[ok])
        den = e.sum(1, keepdims=True)
        out[c0:c0 + 256][ok] = (e[ok] @ v) / den[ok]
    return out


def svg2_attention(q, k, v, Cq: int, Ck: int, iters: int, p: float, scale=None):
    """The whole SVG2 step for one head [L, d]: k-means of Q and K, centroid
    top-p selection, attention under the cluster-pair mask (original order).
    Returns (out, assign_q, assign_k, selected)."""
    aq, mu_q, _ = kmeans(q, Cq, iters)
    ak, mu_k, n_k = kmeans(k, Ck, iters)
    sel = centroid_topp(mu_q, mu_k, n_k, p, scale)
    return svg2_attention_given(q, k, v, aq, ak, sel, scale), aq, ak, sel


def svg2_attention_permuted(q, k, v, assign_q, assign_k, selected, Cq: int, Ck: int, scale=None):
    """The same attention computed the way the page describes the kernel's
    data: Q, K, V permuted so clusters are contiguous, attention over the
    permuted layout with the mask in permuted order, output permuted back."""
    pq, _ = cluster_permutation(assign_q, Cq)
    pk, _ = cluster_permutation(assign_k, Ck)
    qp, kp, vp = np.asarray(q)[pq], np.asarray(k)[pk], np.asarray(v)[pk]
    outp = svg2_attention_given(qp, kp, vp, np.asarray(assign_q)[pq], np.asarray(assign_k)[pk], selected, scale)
    out = np.empty_like(outp)
    out[pq] = outp
    return out
