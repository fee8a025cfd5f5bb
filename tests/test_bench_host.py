"""Host-side logic of bench.py that needs no GPU: the count of (query, key)
pairs the SVG2 cluster-pair attention computes, replayed from the clusters and
the top-p selection, checked against a direct walk of the run rule."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    sys.argv = ["bench.py"]
    import bench
    return bench


def _walk(cid_sorted, keep, nk, rows=256, bk=128):
    """Per CTA of `rows` cluster-sorted query rows: the union of the kept key
    clusters of its query clusters; a run starts at a kept, non-empty cluster
    and extends over kept or empty clusters; each run is cut into bk-key tiles
    computed for all rows of the CTA."""
    Ck = keep.shape[1]
    koff = np.concatenate(([0], np.cumsum(nk)))
    total = 0
    for q0 in range(0, len(cid_sorted), rows):
        c0, c1 = cid_sorted[q0], cid_sorted[min(q0 + rows, len(cid_sorted)) - 1]
        u = [any(keep[c, j] for c in range(c0, c1 + 1)) for j in range(Ck)]
        c = 0
        while True:
            while c < Ck and not (u[c] and nk[c] > 0):
                c += 1
            if c == Ck:
                break
            e = c + 1
            while e < Ck and (u[e] or nk[e] == 0):
                e += 1
            total += -(-(koff[e] - koff[c]) // bk) * bk * rows
            c = e
    return total


@pytest.mark.parametrize("seed", range(6))
def test_s2_computed_pairs_matches_run_walk(seed):
    bench = _bench()
    rng = np.random.default_rng(seed)
    Cq, Ck = int(rng.integers(2, 9)), int(rng.integers(3, 40))
    L = int(rng.integers(300, 2000))
    aq = np.sort(rng.integers(0, Cq, L))
    nk = np.bincount(rng.integers(0, Ck, L), minlength=Ck)
    nk[rng.integers(0, Ck)] = 0  # an empty key cluster
    keep = rng.random((Cq, Ck)) < rng.uniform(0.2, 0.9)
    assert bench.s2_computed_pairs(aq, keep, nk) == _walk(aq, keep, nk)


def test_s2_computed_pairs_dense_and_single_cluster():
    bench = _bench()
    L = 1000
    aq = np.zeros(L, dtype=np.int64)
    nk = np.array([300, 0, 700])
    keep = np.ones((1, 3), dtype=bool)
    # one run of 1000 keys: 8 tiles of 128 for each of the 4 CTAs of 256 rows
    assert bench.s2_computed_pairs(aq, keep, nk) == 4 * 8 * 128 * 256
    keep[0, 2] = False
    # one run of 300 keys (the empty cluster does not extend it): 3 tiles
    assert bench.s2_computed_pairs(aq, keep, nk) == 4 * 3 * 128 * 256
