"""k-nearest-neighbour distogram features -- TEST INFRASTRUCTURE ONLY.

Same import rules as the `oracle` package: only `tests/`,
`__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` may use it;
it imports nothing from the product path.

What it computes ("Flash Invariant Point Attention", rebuttal answer 6 on the
kNN algorithm): instead of the (B, L, L, n_bins) distogram, only the k nearest
neighbours of every residue are kept, (B, L, k, n_bins), and the neighbours
may be found block-wise without an L x L matrix.  Written out plainly here,
one query at a time, with these readings of what the pages leave open:

  * positions are the frame translations (one point per residue);
  * the neighbours of residue i are the k valid residues j of the same sample
    (mask_j true) with the smallest distance |t_j - t_i|, residue i itself
    included (distance 0); a masked query has no neighbours;
  * ties in distance go to the smaller index j; the list is sorted by
    (distance, j); slots beyond the number of valid residues hold index -1,
    distance +inf and bin -1;
  * the squared distance is taken in float32 as ((dx*dx) + (dy*dy)) + (dz*dz)
    with dx = x_j - x_i, each operation rounded to float32 (the precision in
    which the kernel decides the order, so both sides take the same integer
    decisions), and the distance is its correctly rounded float32 sqrt;
  * the distogram bin of a distance d is the number of bin edges e with
    e <= d (edges ascending, n_bins - 1 of them), and the one-hot row of that
    bin is the feature vector (all zero for an empty slot).

Pinned in tests/test_oracle_knn.py against scipy's k-d tree on random points,
closed forms on a line, the tie rule on symmetric configurations, and
numpy's searchsorted for the bins.
"""
from __future__ import annotations

import numpy as np

__all__ = ["knn_distogram", "default_edges"]


def default_edges(n_bins: int, d_min: float = 2.0, d_max: float = 22.0) -> np.ndarray:
    """n_bins - 1 equally spaced float32 edges from d_min to d_max: bin 0 is
    d < d_min, the last bin d >= d_max."""
    return np.linspace(d_min, d_max, n_bins - 1).astype(np.float32)


def knn_distogram(translation, mask, k: int, edges, rows=None) -> dict:
    """translation [B,N,3] (any float dtype; used as float32), mask [B,N] bool,
    edges [n_bins - 1] ascending.  Returns idx [B,R,k] int64, dist [B,R,k]
    float32, bin [B,R,k] int64 and onehot [B,R,k,n_bins] float32 for the query
    rows `rows` (default all)."""
    t = np.asarray(translation, dtype=np.float32)
    m = np.asarray(mask).astype(bool)
    e = np.asarray(edges, dtype=np.float32)
    B, N, _ = t.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    R = len(rows)
    n_bins = len(e) + 1
    idx = np.full((B, R, k), -1, dtype=np.int64)
    dist = np.full((B, R, k), np.inf, dtype=np.float32)
    bins = np.full((B, R, k), -1, dtype=np.int64)
    onehot = np.zeros((B, R, k, n_bins), dtype=np.float32)
    for b in range(B):
        valid = np.flatnonzero(m[b])
        for r, i in enumerate(rows):
            if not m[b, i]:
                continue
            dx = t[b, valid, 0] - t[b, i, 0]
            dy = t[b, valid, 1] - t[b, i, 1]
            dz = t[b, valid, 2] - t[b, i, 2]
            d2 = (dx * dx + dy * dy) + dz * dz            # float32, left to right
            order = np.lexsort((valid, d2))               # by d2, then by index
            take = order[:k]
            n = len(take)
            idx[b, r, :n] = valid[take]
            dist[b, r, :n] = np.sqrt(d2[take])
            bb = np.searchsorted(e, dist[b, r, :n], side="right")
            bins[b, r, :n] = bb
            onehot[b, r, np.arange(n), bb] = 1.0
    return {"idx": idx, "dist": dist, "bin": bins, "onehot": onehot}
