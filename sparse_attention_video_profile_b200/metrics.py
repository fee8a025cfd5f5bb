"""Work accounting for the throughput metric (effective TFLOPS).

Effective work counts only unmasked (query, key) pairs: 4*d flops per pair,
2*d for the q.k dot product and 2*d for the p*v accumulation.  Masked pairs
that a kernel computes inside partially masked tiles are overhead and are not
counted.
"""
from __future__ import annotations

import numpy as np


def band_pairs(n: int, a: int) -> int:
    """Ordered pairs (u, v) on 0..n-1 with |u - v| < a.

    Row u keeps min(n-1, u+a-1) - max(0, u-a+1) + 1 partners; summing over u
    gives n*(2a-1) - a*(a-1) for 1 <= a <= n (a >= n keeps all n*n pairs).
    """
    a = min(a, n)
    return n * (2 * a - 1) - a * (a - 1)


def spatial_pairs(N: int, F: int, a1: int) -> int:
    """Unmasked pairs of the spatial mask |i1 - i2| < a1: frame pairs times F**2
    ("Sparse Video-Gen", Spatial Head)."""
    return F * F * band_pairs(N, a1)


def temporal_pairs(N: int, F: int, a2: int) -> int:
    """Unmasked pairs of the temporal mask |j1 - j2| < a2: position pairs times
    N**2 ("Sparse Video-Gen", Temporal Head)."""
    return N * N * band_pairs(F, a2)


def effective_pairs(N: int, F: int, a1: int, a2: int, labels) -> int:
    """Unmasked pairs summed over heads, each head using its label's mask
    (0 spatial, 1 temporal)."""
    sp = spatial_pairs(N, F, a1)
    tp = temporal_pairs(N, F, a2)
    labels = np.asarray(labels).reshape(-1)
    n_t = int((labels == 1).sum())
    return n_t * tp + (labels.size - n_t) * sp


def attention_flops(pairs: int, d: int) -> float:
    return 4.0 * d * float(pairs)


def window_pairs(L: int, W: int) -> int:
    """Pairs |x - y| <= W on 0..L-1: L*(2W+1) - W*(W+1) for W < L."""
    W = min(W, L - 1)
    return L * (2 * W + 1) - W * (W + 1)


def mixed_pairs(N: int, F: int, modes, window: int, md_half: int, stripe: int) -> int:
    """Unmasked pairs summed over heads of the mixed-pattern call (modes 0 full,
    1 skip, 2 diagonal, 3 multi-diagonal, 4 vertical stripe)."""
    L = N * F
    per = {0: L * L, 1: 0, 2: window_pairs(L, window), 3: temporal_pairs(N, F, md_half + 1),
           4: L * min(stripe, L)}
    return int(sum(per[int(m)] for m in np.asarray(modes).reshape(-1)))
