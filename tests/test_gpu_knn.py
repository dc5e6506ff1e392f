"""The kNN distogram kernel (fipa_knn_distogram, through the C ABI) against the
oracle (oracle/knn.py).  Indices and bins are integer decisions taken in the
same float32 arithmetic on both sides, so every output must be bit-identical:
indices, bins, distances and the one-hot rows ("Flash Invariant Point
Attention", rebuttal answer 6)."""
import numpy as np
import pytest
import torch

import workloads
from oracle.knn import default_edges, knn_distogram

pytestmark = pytest.mark.gpu


def run(trans, mask, k, edges, dtype="f32"):
    from protein_structure_models_b200 import build
    from protein_structure_models_b200.fipa import knn_distogram as gpu_knn
    build.build()
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    t = torch.from_numpy(np.ascontiguousarray(trans)).to(device="cuda", dtype=td)
    m = torch.from_numpy(np.ascontiguousarray(mask).astype(np.uint8)).cuda()
    e = torch.from_numpy(np.asarray(edges, np.float32)).cuda()
    out = gpu_knn(t, m, k, e)
    torch.cuda.synchronize()
    return {key: v.cpu().numpy() for key, v in out.items()}


def check(trans, mask, k, edges, dtype="f32", rows=None):
    got = run(trans, mask, k, edges, dtype)
    ref = knn_distogram(trans, mask, k, edges, rows=rows)
    sl = (slice(None), rows if rows is not None else slice(None))
    np.testing.assert_array_equal(got["idx"][sl], ref["idx"])
    np.testing.assert_array_equal(got["bin"][sl], ref["bin"])
    np.testing.assert_array_equal(got["dist"][sl], ref["dist"])
    np.testing.assert_array_equal(got["onehot"][sl], ref["onehot"])
    return got


def test_random_points_with_masks():
    rng = np.random.default_rng(0)
    t = (rng.standard_normal((3, 300, 3)) * 10).astype(np.float32)
    mask = rng.random((3, 300)) < 0.8
    mask[2, :] = False                                    # a fully masked sample
    check(t, mask, 20, default_edges(16))


def test_ties_on_a_grid():
    """Integer grid points: many exact ties, broken by the smaller index."""
    g = np.stack(np.meshgrid(np.arange(6), np.arange(6), np.arange(6), indexing="ij"), -1).reshape(1, -1, 3)
    t = g.astype(np.float32)
    check(t, np.ones((1, t.shape[1]), bool), 27, default_edges(8, 0.5, 3.5))


@pytest.mark.parametrize("k", [1, 32])
def test_k_extremes_and_short_samples(k):
    rng = np.random.default_rng(k)
    t = (rng.standard_normal((4, 21, 3)) * 4).astype(np.float32)
    mask = np.ones((4, 21), bool)
    mask[1, 5:] = False                                   # fewer valid residues than k
    check(t, mask, k, default_edges(4))


def test_single_residue_and_single_bin():
    t = np.zeros((2, 1, 3), np.float32)
    check(t, np.array([[True], [False]]), 5, np.zeros(0, np.float32))


def test_short_chain_batch_bf16():
    """Random-walk translations of the short-chain batch (bf16, lengths U{40..150})."""
    inp = workloads.make_inputs(workloads.workload(4).with_(B=16))
    check(inp["translation"], inp["mask"], 20, default_edges(39, 3.25, 50.75), dtype="bf16")


def test_long_chain_sampled_rows():
    """The 16384-residue chain (several key blocks per CTA), 96 sampled query rows."""
    inp = workloads.make_inputs(workloads.workload("3-16384"))
    rows = np.unique(np.concatenate([[0, 2047, 2048, 16383], np.random.default_rng(3).choice(16384, 92, replace=False)]))
    check(inp["translation"], inp["mask"], 20, default_edges(39, 3.25, 50.75), dtype="bf16", rows=rows)
