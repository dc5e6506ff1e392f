"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Every check follows the BioTorch page "Invariant point attention (IPA)",
section "Required behavior", unless it says otherwise.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
from scipy.spatial import distance
from scipy.spatial.transform import Rotation

import oracle
from oracle.bruteforce import ipa_bruteforce
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_inputs(seed=0, B=2, N=6, H=2, D=3, Dv=2, P=2, Q=2, Cz=3, R=2, Cout=4,
                 empty_row=True, t_scale=4.0):
    """Random float64 inputs with masks, including one empty neighbourhood."""
    rng = np.random.default_rng(seed)
    g = rng.standard_normal
    F = H * (Dv + 4 * Q + Cz)
    inp = dict(q=g((B, N, H, D)), k=g((B, N, H, D)), v=g((B, N, H, Dv)),
               q_points=g((B, N, H, P, 3)), k_points=g((B, N, H, P, 3)),
               v_points=g((B, N, H, Q, 3)),
               rotation=workloads.random_rotations(rng, (B, N)),
               translation=t_scale * g((B, N, 3)),
               z1=g((B, N, R, Cz)), z2=g((B, N, R, Cz)), Wb=g((Cz, H)),
               point_weight_raw=g((H,)), w_out=g((F, Cout)) / math.sqrt(F),
               b_out=g((Cout,)), eps=1e-8)
    mask = rng.random((B, N)) < 0.8
    mask[:, 0] = True
    pair_mask = rng.random((B, N, N)) < 0.85
    if empty_row:
        pair_mask[0, 0, :] = False        # query 0 of sample 0: empty neighbourhood
    inp["mask"] = mask
    inp["pair_mask"] = pair_mask
    return inp


# --------------------------------------------------------------------------
# worked example "Nearby frames receive more weight": closed form
# --------------------------------------------------------------------------
def _worked_example_inputs(fx, d):
    pr = fx["printed_on_page"]
    act = {
        "q": np.zeros((1, 2, 1, 1)), "k": np.zeros((1, 2, 1, 1)),
        "v": np.array(pr["v"], float).reshape(1, 2, 1, 1),
        "q_points": np.zeros((1, 2, 1, 1, 3)), "k_points": np.zeros((1, 2, 1, 1, 3)),
        "v_points": np.tile(np.array([1.0, 0, 0]), (1, 2, 1, 1, 1)),
        "pair_bias": np.zeros((1, 2, 2, 1)),
        "pair_values": np.array(pr["pair_values_query_key"], float).reshape(1, 2, 2, 1),
    }
    par = {"point_weight_raw": np.zeros(1), "w_out": np.array(pr["w_out"], float),
           "b_out": np.array(pr["b_out"], float)}
    masks = {"mask": np.ones((1, 2), bool), "pair_mask": np.ones((1, 2, 2), bool)}
    struct = {"rotation": np.tile(np.eye(3), (1, 2, 1, 1)),
              "translation": np.array([[[0.0, 0, 0], [d, 0, 0]]])}
    return act, par, masks, struct, float(pr["eps"])


def _worked_example_closed_form(d, eps):
    # L_00 = L_11 = 0 and L_01 = L_10 = -c d^2 with c = 1/2 ln2 sqrt(2/27)
    # (softplus(0) = ln 2, P = 1); softmax of two logits is a logistic sigmoid.
    c = 0.5 * math.log(2.0) * math.sqrt(2.0 / 27.0)
    a_self = 1.0 / (1.0 + math.exp(-c * d * d))
    a_other = 1.0 - a_self
    upd = [3 * a_self + 9 * a_other,          # (2 a00 + 6 a01) + (1 a00 + 3 a01)
           6 * a_other + 8 * a_self]          # (2 a10 + 6 a11) + (4 a10 + 2 a11)
    loc_x = [1.0 + a_other * d, 1.0 - a_other * d]
    return a_self, upd, loc_x


@pytest.mark.parametrize("d", [1.0, 3.0, 6.0])
def test_worked_example_closed_form(d):
    with open(os.path.join(GOLDEN, "worked_example_nearby_frames.json")) as f:
        fx = json.load(f)
    act, par, masks, struct, eps = _worked_example_inputs(fx, d)
    out = oracle.invariant_point_attention(act, par, masks, struct, eps=eps)
    a_self, upd, loc_x = _worked_example_closed_form(d, eps)
    att = out["attention"][0, 0]
    assert att[0, 0] == pytest.approx(a_self, abs=1e-14)
    assert att[1, 1] == pytest.approx(a_self, abs=1e-14)
    assert att[0, 1] == pytest.approx(1 - a_self, abs=1e-14)
    # "nearby frames receive more weight"
    assert att[0, 0] > att[0, 1] and att[1, 1] > att[1, 0]
    np.testing.assert_allclose(out["update"][0, :, 0], upd, atol=1e-13)
    np.testing.assert_allclose(out["local_points"][0, :, 0, 0, 0], loc_x, atol=1e-13)
    np.testing.assert_allclose(out["local_points"][0, :, 0, 0, 1:], 0.0, atol=1e-15)


@pytest.mark.parametrize("d", [1.0, 3.0])
def test_worked_example_through_factors(d):
    """The same example given as factors z1, z2 (R=2, Cz=1) and Wb = 0."""
    with open(os.path.join(GOLDEN, "worked_example_nearby_frames.json")) as f:
        fx = json.load(f)
    act, par, masks, struct, eps = _worked_example_inputs(fx, d)
    pv = act["pair_values"][0, :, :, 0]
    inp = {k: act[k] for k in ("q", "k", "v", "q_points", "k_points", "v_points")}
    inp.update(par)
    inp.update(struct)
    inp.update(mask=masks["mask"], pair_mask=None, eps=eps,
               z1=pv.reshape(1, 2, 2, 1), z2=np.eye(2).reshape(1, 2, 2, 1),
               Wb=np.zeros((1, 1)))
    a_self, upd, loc_x = _worked_example_closed_form(d, eps)
    for fn in (oracle.ipa_forward_dense, oracle.ipa_forward_factorised):
        out = fn(inp, want_attention=True)
        np.testing.assert_allclose(out["update"][0, :, 0], upd, atol=1e-13)
        np.testing.assert_allclose(out["local_points"][0, :, 0, 0, 0], loc_x, atol=1e-13)
        assert out["attention"][0, 0, 0, 0] == pytest.approx(a_self, abs=1e-14)


# --------------------------------------------------------------------------
# softplus without overflow
# --------------------------------------------------------------------------
def test_softplus_matches_logaddexp_without_overflow():
    x = np.concatenate([np.linspace(-800, 800, 4001), [-1e300, 1e300, 0.0]])
    with np.errstate(over="raise", invalid="raise"):
        y = oracle.softplus(x)
    ref = np.logaddexp(0.0, x)
    np.testing.assert_allclose(y, ref, rtol=1e-15, atol=1e-300)
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), abs=1e-16)


# --------------------------------------------------------------------------
# SE(3) invariance under a common global motion
# --------------------------------------------------------------------------
def _moved(inp, seed):
    rng = np.random.default_rng(seed)
    G = workloads.random_rotations(rng, ())
    u = 50.0 * rng.standard_normal(3)
    out = dict(inp)
    out["rotation"] = np.einsum("xy,bnyz->bnxz", G, inp["rotation"])
    out["translation"] = np.einsum("xy,bny->bnx", G, inp["translation"]) + u
    return out


def _assert_same_outputs(a, b, tol=1e-9):
    for key in ("update", "local_points", "attention"):
        np.testing.assert_allclose(a[key], b[key], rtol=tol, atol=tol)
    fin = np.isfinite(a["lse"])
    assert np.array_equal(fin, np.isfinite(b["lse"]))
    np.testing.assert_allclose(a["lse"][fin], b["lse"][fin], rtol=tol, atol=tol)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_rigid_motion_invariance(seed):
    inp = small_inputs(seed, N=7)
    base = oracle.ipa_forward_dense(inp, want_attention=True)
    moved = oracle.ipa_forward_dense(_moved(inp, 100 + seed), want_attention=True)
    _assert_same_outputs(base, moved)


def test_rigid_motion_invariance_workload0():
    inp = workloads.make_inputs(workloads.workload(0))
    base = oracle.ipa_forward_dense(inp, want_attention=True)
    moved = oracle.ipa_forward_dense(_moved(inp, 7), want_attention=True)
    _assert_same_outputs(base, moved, tol=1e-8)


# --------------------------------------------------------------------------
# softmax rows, masks, empty neighbourhoods
# --------------------------------------------------------------------------
def test_rows_sum_to_one_or_zero_and_structural_zeros():
    inp = small_inputs(3, B=2, N=8)
    out = oracle.ipa_forward_dense(inp, want_attention=True)
    att = out["attention"]                                  # [B,H,N,N]
    permitted = (inp["mask"][:, :, None] & inp["mask"][:, None, :] & inp["pair_mask"])
    # not-permitted entries are exactly zero
    assert np.all(att[np.broadcast_to(~permitted[:, None], att.shape)] == 0.0)
    sums = att.sum(-1)
    empty = ~permitted.any(-1)                              # [B,N]
    assert empty[0, 0]
    for b in range(att.shape[0]):
        for i in range(att.shape[2]):
            if empty[b, i]:
                assert np.all(sums[b, :, i] == 0.0)
                assert np.all(out["update"][b, i] == 0.0)      # not b_out
                assert np.all(out["local_points"][b, i] == 0.0)
                assert np.all(np.isneginf(out["lse"][b, :, i]))
            else:
                np.testing.assert_allclose(sums[b, :, i], 1.0, atol=1e-12)


def test_masked_query_is_empty_neighbourhood():
    inp = small_inputs(4, empty_row=False)
    inp["mask"][1, 3] = False
    out = oracle.ipa_forward_dense(inp, want_attention=True)
    assert np.all(out["update"][1, 3] == 0.0)
    assert np.all(out["local_points"][1, 3] == 0.0)
    assert np.all(out["attention"][1, :, 3, :] == 0.0)


# --------------------------------------------------------------------------
# special cases that reduce to library routines
# --------------------------------------------------------------------------
def test_scalar_only_reduces_to_sdpa():
    """Points and translations zero, pair factors zero: the attention is a
    masked softmax(q k^T / sqrt(3D)); checked with torch's SDPA (fp64, CPU)."""
    import torch
    inp = small_inputs(5, B=2, N=8, H=3, D=4, Dv=5, P=2, Q=2, Cz=2, empty_row=False)
    B, N, H, D = inp["q"].shape
    Dv = inp["v"].shape[-1]
    F = H * (Dv + 4 * 2 + 2)
    inp["q_points"][:] = 0
    inp["k_points"][:] = 0
    inp["translation"][:] = 0
    inp["z1"][:] = 0
    inp["pair_mask"] = None
    w = np.zeros((F, H * Dv))
    w[:H * Dv, :] = np.eye(H * Dv)                  # update = scalar block of features
    inp["w_out"], inp["b_out"] = w, np.zeros(H * Dv)
    out = oracle.ipa_forward_dense(inp, want_attention=True)
    tq = torch.from_numpy(inp["q"]).permute(0, 2, 1, 3)
    tk = torch.from_numpy(inp["k"]).permute(0, 2, 1, 3)
    tv = torch.from_numpy(inp["v"]).permute(0, 2, 1, 3)
    m = torch.from_numpy(inp["mask"])
    am = (m[:, None, :, None] & m[:, None, None, :])
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=am, scale=1.0 / math.sqrt(3 * D)).permute(0, 2, 1, 3).numpy()
    for b in range(B):
        for i in range(N):
            if inp["mask"][b, i]:
                np.testing.assert_allclose(out["update"][b, i].reshape(H, Dv), ref[b, i], atol=1e-12)
            else:
                assert np.all(out["update"][b, i] == 0)


def test_distance_only_matches_cdist_softmax():
    """q = k = 0 and zero pair factors: logits are -gamma_h times the squared
    distance of the stacked global points; global points via scipy Rotation,
    distances via scipy cdist, softmax / logsumexp via scipy.special."""
    inp = small_inputs(6, B=1, N=8, H=3, P=3, empty_row=False)
    inp["q"][:] = 0
    inp["k"][:] = 0
    inp["z1"][:] = 0
    out = oracle.ipa_forward_dense(inp, want_attention=True)
    B, N, H, P, _ = inp["q_points"].shape
    rot = Rotation.from_matrix(inp["rotation"][0])
    gamma = 0.5 * np.logaddexp(0.0, inp["point_weight_raw"]) * math.sqrt(2.0 / (27 * P))
    permitted = inp["mask"][0][:, None] & inp["mask"][0][None, :] & inp["pair_mask"][0]
    for h in range(H):
        A = np.stack([rot[i].apply(inp["q_points"][0, i, h]) + inp["translation"][0, i]
                      for i in range(N)]).reshape(N, 3 * P)
        Bk = np.stack([rot[j].apply(inp["k_points"][0, j, h]) + inp["translation"][0, j]
                       for j in range(N)]).reshape(N, 3 * P)
        logits = -gamma[h] * distance.cdist(A, Bk, "sqeuclidean")
        for i in range(N):
            if not permitted[i].any():
                continue
            row = np.where(permitted[i], logits[i], -np.inf)
            np.testing.assert_allclose(out["attention"][0, h, i], scipy.special.softmax(row), atol=1e-12)
            assert out["lse"][0, h, i] == pytest.approx(scipy.special.logsumexp(row), abs=1e-10)


def test_identity_neighbourhood_closed_form():
    """pair_mask = I: attention = I; local point = R_i^T (R_i v + t_i - t_i) = v;
    the features are then known in closed form."""
    inp = small_inputs(7, B=1, N=5, H=2, Dv=2, Q=3, Cz=2, empty_row=False)
    B, N, H, Q = 1, 5, 2, 3
    inp["mask"][:] = True
    inp["pair_mask"] = np.broadcast_to(np.eye(N, dtype=bool), (B, N, N)).copy()
    out = oracle.ipa_forward_dense(inp, want_attention=True)
    np.testing.assert_array_equal(out["attention"][0], np.broadcast_to(np.eye(N), (H, N, N)))
    np.testing.assert_allclose(out["local_points"], inp["v_points"], atol=1e-12)
    vp = inp["v_points"][0]
    zdiag = np.einsum("irc,irc->ic", inp["z1"][0], inp["z2"][0])
    feats = np.concatenate([inp["v"][0].reshape(N, -1), vp[..., 0].reshape(N, -1),
                            vp[..., 1].reshape(N, -1), vp[..., 2].reshape(N, -1),
                            np.sqrt((vp ** 2).sum(-1) + inp["eps"]).reshape(N, -1),
                            np.repeat(zdiag[:, None, :], H, axis=1).reshape(N, -1)], axis=1)
    np.testing.assert_allclose(out["update"][0], feats @ inp["w_out"] + inp["b_out"], atol=1e-12)


def test_feature_blocks_head_major():
    """With w_out = identity the update IS the feature vector: its x/y/z/length
    blocks must be the local points flattened (head, point)."""
    inp = small_inputs(8, B=1, N=6, H=3, Dv=2, Q=2, Cz=2, empty_row=False)
    H, Dv, Q, Cz = 3, 2, 2, 2
    F = H * (Dv + 4 * Q + Cz)
    inp["w_out"], inp["b_out"] = np.eye(F), np.zeros(F)
    out = oracle.ipa_forward_dense(inp)
    lp = out["local_points"][0]                               # [N,H,Q,3]
    u = out["update"][0]
    o = H * Dv
    for x in range(3):
        blk = u[:, o + x * H * Q: o + (x + 1) * H * Q]
        live = inp["mask"][0]
        np.testing.assert_allclose(blk[live], lp[live][..., x].reshape(-1, H * Q), atol=1e-13)
    lenblk = u[:, o + 3 * H * Q: o + 4 * H * Q]
    live = inp["mask"][0]
    np.testing.assert_allclose(lenblk[live], np.sqrt((lp[live] ** 2).sum(-1) + inp["eps"]).reshape(-1, H * Q), atol=1e-13)


# --------------------------------------------------------------------------
# brute force and the second arithmetic path
# --------------------------------------------------------------------------
@pytest.mark.parametrize("seed,N", [(10, 4), (11, 6), (12, 8)])
def test_bruteforce_agrees(seed, N):
    inp = small_inputs(seed, B=2, N=N)
    vec = oracle.ipa_forward_dense(inp, want_attention=True)
    bf = ipa_bruteforce(inp)
    np.testing.assert_allclose(vec["update"], np.array(bf["update"]), atol=1e-11)
    np.testing.assert_allclose(vec["local_points"], np.array(bf["local_points"]), atol=1e-11)
    np.testing.assert_allclose(vec["attention"], np.array(bf["attention"]), atol=1e-12)


@pytest.mark.parametrize("seed", [20, 21])
def test_dense_equals_factorised(seed):
    inp = small_inputs(seed, B=2, N=8, H=3, Cz=5, R=3)
    a = oracle.ipa_forward_dense(inp, want_attention=True)
    b = oracle.ipa_forward_factorised(inp, want_attention=True)
    _assert_same_outputs(a, b, tol=1e-12)


def test_dense_equals_factorised_walk_workload():
    wl = workloads.workload(1).with_(B=2, N=40, Cz=16, Cout=8)
    inp = workloads.make_inputs(wl)
    a = oracle.ipa_forward_dense(inp, want_attention=True)
    b = oracle.ipa_forward_factorised(inp, want_attention=True)
    _assert_same_outputs(a, b, tol=1e-10)


def test_row_subset_is_exact():
    wl = workloads.workload(1).with_(B=2, N=48, Cz=16, Cout=8)
    inp = workloads.make_inputs(wl)
    full = oracle.ipa_forward_dense(inp, want_attention=True)
    rows = [0, 5, 47, 13]
    sub = oracle.ipa_forward_dense(inp, rows=rows, want_attention=True)
    np.testing.assert_array_equal(sub["update"], full["update"][:, rows])
    np.testing.assert_array_equal(sub["attention"], full["attention"][:, :, rows])


# --------------------------------------------------------------------------
# the pins catch planted mistakes (planted in the oracle, on the CPU)
# --------------------------------------------------------------------------
def test_planted_transposed_rotation_is_caught(monkeypatch):
    def wrong_frames(rotation, translation, points):
        return (np.einsum("...nyx,...nhpy->...nhpx", rotation, points)
                + translation[..., :, None, None, :])
    monkeypatch.setattr(oracle, "apply_frames", wrong_frames)
    inp = small_inputs(30, N=7)
    base = oracle.ipa_forward_dense(inp, want_attention=True)
    moved = oracle.ipa_forward_dense(_moved(inp, 31), want_attention=True)
    with pytest.raises(AssertionError):
        _assert_same_outputs(base, moved)


def test_planted_distance_sign_is_caught(monkeypatch):
    real = oracle.point_weight
    monkeypatch.setattr(oracle, "point_weight", lambda raw, P: -real(raw, P))
    with open(os.path.join(GOLDEN, "worked_example_nearby_frames.json")) as f:
        fx = json.load(f)
    act, par, masks, struct, eps = _worked_example_inputs(fx, 3.0)
    out = oracle.invariant_point_attention(act, par, masks, struct, eps=eps)
    a_self, _, _ = _worked_example_closed_form(3.0, eps)
    assert abs(out["attention"][0, 0, 0, 0] - a_self) > 0.1


def test_planted_missing_point_scale_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "point_weight", lambda raw, P: 0.5 * oracle.softplus(raw))
    with open(os.path.join(GOLDEN, "worked_example_nearby_frames.json")) as f:
        fx = json.load(f)
    act, par, masks, struct, eps = _worked_example_inputs(fx, 3.0)
    out = oracle.invariant_point_attention(act, par, masks, struct, eps=eps)
    a_self, _, _ = _worked_example_closed_form(3.0, eps)
    assert abs(out["attention"][0, 0, 0, 0] - a_self) > 0.05


# --------------------------------------------------------------------------
# the pair-bias term alone: closed form (logit bullet, pair_bias / sqrt(3))
# --------------------------------------------------------------------------
def _sigmoid(x):
    return 1.0 / (1.0 + math.exp(-x))


def _pair_bias_case(Wb_override=None):
    """Two residues, identity frames at the origin, q = k = points = 0: the only
    non-zero logit term is pair_bias / sqrt(3) (tests/golden/pair_bias_two_residues.json)."""
    with open(os.path.join(GOLDEN, "pair_bias_two_residues.json")) as f:
        fx = json.load(f)
    B, N, H, D, Dv, P, Q, Cz, R = (fx[k] for k in ("B", "N", "H", "D", "Dv", "P", "Q", "Cz", "R"))
    F = H * (Dv + 4 * Q + Cz)
    inp = dict(q=np.zeros((B, N, H, D)), k=np.zeros((B, N, H, D)), v=np.ones((B, N, H, Dv)),
               q_points=np.zeros((B, N, H, P, 3)), k_points=np.zeros((B, N, H, P, 3)),
               v_points=np.zeros((B, N, H, Q, 3)),
               rotation=np.tile(np.eye(3), (B, N, 1, 1)), translation=np.zeros((B, N, 3)),
               z1=np.array(fx["z1_i_r_c"], float)[None], z2=np.array(fx["z2_j_r_c"], float)[None],
               Wb=np.array(fx["Wb_c_h"], float) if Wb_override is None else Wb_override,
               point_weight_raw=np.zeros(H), w_out=np.eye(F), b_out=np.zeros(F), eps=1e-8,
               mask=np.ones((B, N), bool), pair_mask=None)
    s3 = math.sqrt(3.0)
    # hand-computed biases b_ij,h: b00 = (3, 1), b11 = (1, 4), b01 = b10 = 0
    a = {(0, 0): _sigmoid(3 / s3), (1, 0): _sigmoid(1 / s3),      # (h, i): a[h][i][i]
         (0, 1): _sigmoid(1 / s3), (1, 1): _sigmoid(4 / s3)}
    pair_feat = np.array([[a[0, 0], 0.0, a[1, 0], 0.0],
                          [0.0, 2 * a[0, 1], 0.0, 2 * a[1, 1]]])
    return inp, a, pair_feat


def test_pair_bias_closed_form_through_factors():
    inp, a, pair_feat = _pair_bias_case()
    for fn in (oracle.ipa_forward_dense, oracle.ipa_forward_factorised):
        out = fn(inp, want_attention=True)
        att = out["attention"][0]                          # [H, N, N]
        for (h, i), val in a.items():
            assert att[h, i, i] == pytest.approx(val, abs=1e-14)
            assert att[h, i, 1 - i] == pytest.approx(1 - val, abs=1e-14)
        np.testing.assert_allclose(out["update"][0][:, 10:14], pair_feat, atol=1e-14)


def test_pair_bias_closed_form_through_page_signature():
    """The same case through the page's dense signature: pair_bias [B,N,N,H] and
    pair_values [B,N,N,Cz] written out by hand."""
    inp, a, pair_feat = _pair_bias_case()
    pb = np.zeros((1, 2, 2, 2))
    pb[0, 0, 0] = [3.0, 1.0]
    pb[0, 1, 1] = [1.0, 4.0]
    pv = np.zeros((1, 2, 2, 2))
    pv[0, 0, 0] = [1.0, 0.0]
    pv[0, 1, 1] = [0.0, 2.0]
    act = {k: inp[k] for k in ("q", "k", "v", "q_points", "k_points", "v_points")}
    act.update(pair_bias=pb, pair_values=pv)
    par = {k: inp[k] for k in ("point_weight_raw", "w_out", "b_out")}
    out = oracle.invariant_point_attention(act, par, {"mask": inp["mask"], "pair_mask": None},
                                           {"rotation": inp["rotation"], "translation": inp["translation"]},
                                           eps=inp["eps"])
    for (h, i), val in a.items():
        assert out["attention"][0, h, i, i] == pytest.approx(val, abs=1e-14)
    np.testing.assert_allclose(out["update"][0][:, 10:14], pair_feat, atol=1e-14)


@pytest.mark.parametrize("plant", ["Wb transposed", "missing 1/sqrt(3)"])
def test_pair_bias_pin_catches_planted_mistakes(plant):
    """A transposed projection or a bias without its 1/sqrt(3) moves the
    attention by far more than rounding (planted through the inputs)."""
    Wb = np.array([[3.0, 1.0], [0.5, 2.0]])
    wrong = Wb.T.copy() if plant == "Wb transposed" else Wb * math.sqrt(3.0)
    inp, a, _ = _pair_bias_case(Wb_override=wrong)
    att = oracle.ipa_forward_dense(inp, want_attention=True)["attention"][0]
    worst = max(abs(att[h, i, i] - val) for (h, i), val in a.items())
    assert worst > 0.05, worst


# --------------------------------------------------------------------------
# eps inside the output point lengths: worked example, length column of w_out
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d", [0.0, 1.0, 3.0])
def test_worked_example_lengths_with_eps(d):
    """The page's worked example (eps = 1) with w_out picking the point-length
    feature: update_i = sqrt(local_x_i^2 + eps), local_x = (1 + a_01 d, 1 - a_10 d)
    and local y = z = 0.  At d = 0 the length is sqrt(2), not 1: eps is inside
    the root ("used inside the OUTPUT point-length square root")."""
    with open(os.path.join(GOLDEN, "worked_example_nearby_frames.json")) as f:
        fx = json.load(f)
    act, par, masks, struct, eps = _worked_example_inputs(fx, d)
    assert eps == 1.0
    par = dict(par, w_out=np.array([[0.0], [0.0], [0.0], [0.0], [1.0], [0.0]]))
    out = oracle.invariant_point_attention(act, par, masks, struct, eps=eps)
    _, _, loc_x = _worked_example_closed_form(d, eps)
    want = [math.sqrt(x * x + 1.0) for x in loc_x]
    np.testing.assert_allclose(out["update"][0, :, 0], want, atol=1e-13)
    if d == 0.0:
        np.testing.assert_allclose(out["update"][0, :, 0], math.sqrt(2.0), atol=1e-15)
