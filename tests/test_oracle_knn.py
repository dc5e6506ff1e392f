"""Pins of the kNN distogram oracle (oracle/knn.py) against what does not share
its code: scipy's k-d tree, closed forms on a line, the tie rule on symmetric
configurations, and the bin rule ("Flash Invariant Point Attention", rebuttal
answer 6: keep (B, L, k, n_bins) instead of (B, L, L, n_bins))."""
import numpy as np
import pytest
from scipy.spatial import cKDTree

from oracle.knn import default_edges, knn_distogram


def test_matches_kdtree_on_random_points():
    rng = np.random.default_rng(0)
    t = (rng.standard_normal((2, 300, 3)) * 10).astype(np.float32)
    mask = np.ones((2, 300), bool)
    out = knn_distogram(t, mask, 20, default_edges(16))
    for b in range(2):
        d, j = cKDTree(t[b].astype(np.float64)).query(t[b].astype(np.float64), k=20)
        np.testing.assert_array_equal(out["idx"][b], j)
        np.testing.assert_allclose(out["dist"][b], d, rtol=2e-6, atol=1e-6)
    assert np.all(out["idx"][:, :, 0] == np.arange(300))          # itself first, distance 0
    assert np.all(out["dist"][:, :, 0] == 0.0)


def test_masked_residues_are_not_neighbours_and_have_none():
    rng = np.random.default_rng(1)
    t = (rng.standard_normal((1, 50, 3)) * 5).astype(np.float32)
    mask = rng.random((1, 50)) < 0.6
    out = knn_distogram(t, mask, 8, default_edges(8))
    valid = np.flatnonzero(mask[0])
    tree = cKDTree(t[0, valid].astype(np.float64))
    for i in range(50):
        if not mask[0, i]:
            assert np.all(out["idx"][0, i] == -1) and np.all(np.isinf(out["dist"][0, i]))
            assert np.all(out["onehot"][0, i] == 0)
            continue
        d, jj = tree.query(t[0, i].astype(np.float64), k=8)
        np.testing.assert_array_equal(out["idx"][0, i], valid[jj])


def test_line_closed_form_and_tie_rule():
    """Residues at x = 0, 1, ..., 9 on a line: the neighbours of i are i, then
    i-1 before i+1 (same distance, smaller index first), i-2, i+2, ..."""
    t = np.zeros((1, 10, 3), np.float32)
    t[0, :, 0] = np.arange(10)
    out = knn_distogram(t, np.ones((1, 10), bool), 5, default_edges(4, 0.5, 2.5))
    np.testing.assert_array_equal(out["idx"][0, 5], [5, 4, 6, 3, 7])
    np.testing.assert_array_equal(out["dist"][0, 5], [0, 1, 1, 2, 2])
    np.testing.assert_array_equal(out["idx"][0, 0], [0, 1, 2, 3, 4])
    np.testing.assert_array_equal(out["idx"][0, 9], [9, 8, 7, 6, 5])
    # edges 0.5, 1.5, 2.5: d = 0 -> bin 0, 1 -> 1, 2 -> 2, 3 -> 3
    np.testing.assert_array_equal(out["bin"][0, 0], [0, 1, 2, 3, 3])


def test_fewer_valid_residues_than_k():
    t = np.zeros((1, 3, 3), np.float32)
    t[0, :, 1] = [0, 4, 9]
    out = knn_distogram(t, np.ones((1, 3), bool), 5, default_edges(3, 1.0, 5.0))
    np.testing.assert_array_equal(out["idx"][0, 1], [1, 0, 2, -1, -1])
    assert np.all(np.isinf(out["dist"][0, 1, 3:])) and np.all(out["bin"][0, 1, 3:] == -1)
    np.testing.assert_array_equal(out["bin"][0, 1, :3], [0, 1, 2])   # 0 < 1; 1 <= 4 < 5; 5 <= 5


def test_bins_against_searchsorted_and_onehot():
    rng = np.random.default_rng(2)
    t = (rng.standard_normal((1, 64, 3)) * 8).astype(np.float32)
    edges = default_edges(39, 3.25, 50.75)
    out = knn_distogram(t, np.ones((1, 64), bool), 20, edges)
    d = out["dist"][0]
    want = np.array([[np.sum(edges <= x) for x in row] for row in d])
    np.testing.assert_array_equal(out["bin"][0], want)
    assert np.all(out["onehot"].sum(-1) == 1.0)
    np.testing.assert_array_equal(out["onehot"][0].argmax(-1), want)


def test_tie_rule_is_pinned_by_exact_ties():
    """On the line every pair of neighbours at +-d ties exactly in float32; a
    rule that put the larger index first would give [5, 6, 4], which the line
    closed form above rejects."""
    t = np.zeros((1, 10, 3), np.float32)
    t[0, :, 0] = np.arange(10)
    out = knn_distogram(t, np.ones((1, 10), bool), 3, default_edges(4))
    assert out["dist"][0, 5, 1] == out["dist"][0, 5, 2]
    np.testing.assert_array_equal(out["idx"][0, 5], [5, 4, 6])
