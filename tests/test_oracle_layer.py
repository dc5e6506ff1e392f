"""Pins of the IPA-layer oracle (oracle/layer.py): reduction to the core,
the quaternion frame update against scipy's rotations, and the behaviour of
the layer under a global rigid motion (page "Invariant point attention
(IPA)", Required behavior: the core's outputs are invariant)."""
import math

import numpy as np
import pytest
from scipy.spatial.transform import Rotation

import oracle
import workloads
from oracle.layer import ipa_layer, layer_widths, quaternion_rotation

DIMS = dict(H=2, D=3, Dv=2, P=2, Q=2, Cz=3, R=2)


def layer_inputs(seed=0, B=2, N=7, Cs=12, dims=DIMS):
    rng = np.random.default_rng(seed)
    H, Dv, Q, Cz = dims["H"], dims["Dv"], dims["Q"], dims["Cz"]
    _, Din = layer_widths(**dims)
    F = H * (Dv + 4 * Q + Cz)
    g = rng.standard_normal
    mask = rng.random((B, N)) < 0.85
    mask[:, 0] = True
    return dict(s=g((B, N, Cs)), W_in=g((Cs, Din)) / math.sqrt(Cs), b_in=0.1 * g(Din),
                rotation=workloads.random_rotations(rng, (B, N)), translation=4.0 * g((B, N, 3)),
                mask=mask, pair_mask=None, Wb=g((Cz, H)), point_weight_raw=g(H),
                w_out=g((F, Cs)) / math.sqrt(F), b_out=g(Cs), W_bb=0.1 * g((Cs, 6)), b_bb=0.1 * g(6), eps=1e-8)


def test_quaternion_rotation_matches_scipy():
    rng = np.random.default_rng(1)
    bcd = rng.standard_normal((20, 3))
    got = quaternion_rotation(bcd[:, 0], bcd[:, 1], bcd[:, 2])
    want = Rotation.from_quat(np.concatenate([bcd, np.ones((20, 1))], 1)).as_matrix()   # (x, y, z, w)
    np.testing.assert_allclose(got, want, atol=1e-14)
    np.testing.assert_allclose(quaternion_rotation(0.0, 0.0, 0.0), np.eye(3), atol=0)


def test_reduces_to_the_core_with_selecting_weights():
    """s = the core's inputs laid side by side and W_in = identity: X = s, the
    core sees exactly those inputs, so s' - s is the core's update."""
    inp = layer_inputs(2)
    B, N = inp["s"].shape[:2]
    _, Din = layer_widths(**DIMS)
    Cs = Din
    rng = np.random.default_rng(3)
    F = DIMS["H"] * (DIMS["Dv"] + 4 * DIMS["Q"] + DIMS["Cz"])
    inp.update(s=rng.standard_normal((B, N, Cs)), W_in=np.eye(Cs), b_in=np.zeros(Cs),
               w_out=rng.standard_normal((F, Cs)) / math.sqrt(F), b_out=rng.standard_normal(Cs),
               W_bb=np.zeros((Cs, 6)), b_bb=np.zeros(6))
    out = ipa_layer(inp, DIMS)
    core = oracle.ipa_forward_dense(out["core_inputs"])
    np.testing.assert_allclose(out["s"] - inp["s"], core["update"], atol=1e-12)
    np.testing.assert_array_equal(out["core_inputs"]["q"].reshape(B, N, -1), inp["s"][..., :DIMS["H"] * DIMS["D"]])
    np.testing.assert_allclose(out["rotation"], inp["rotation"], atol=0)      # zero frame update
    np.testing.assert_allclose(out["translation"], inp["translation"], atol=0)


def test_constant_frame_update_composes_on_the_right():
    inp = layer_inputs(4)
    inp["W_bb"] = np.zeros_like(inp["W_bb"])
    inp["b_bb"] = np.array([0.3, -0.2, 0.5, 1.0, 2.0, -0.5])
    out = ipa_layer(inp, DIMS)
    dR = Rotation.from_quat([0.3, -0.2, 0.5, 1.0]).as_matrix()
    live = inp["mask"]
    want_R = np.einsum("bnxy,yz->bnxz", inp["rotation"], dR)
    want_t = np.einsum("bnxy,y->bnx", inp["rotation"], [1.0, 2.0, -0.5]) + inp["translation"]
    np.testing.assert_allclose(out["rotation"][live], want_R[live], atol=1e-12)
    np.testing.assert_allclose(out["translation"][live], want_t[live], atol=1e-12)
    np.testing.assert_array_equal(out["rotation"][~live], inp["rotation"][~live])    # masked: unchanged


@pytest.mark.parametrize("seed", [5, 6])
def test_rigid_motion(seed):
    """A global motion (G, u) of the input frames leaves s' unchanged and moves
    the new frames with it: R'' = G R', t'' = G t' + u."""
    inp = layer_inputs(seed)
    rng = np.random.default_rng(100 + seed)
    G = workloads.random_rotations(rng, ())
    u = 10.0 * rng.standard_normal(3)
    moved = dict(inp, rotation=np.einsum("xy,bnyz->bnxz", G, inp["rotation"]),
                 translation=np.einsum("xy,bny->bnx", G, inp["translation"]) + u)
    a, b = ipa_layer(inp, DIMS), ipa_layer(moved, DIMS)
    np.testing.assert_allclose(b["s"], a["s"], atol=1e-10)
    np.testing.assert_allclose(b["rotation"], np.einsum("xy,bnyz->bnxz", G, a["rotation"]), atol=1e-10)
    np.testing.assert_allclose(b["translation"], np.einsum("xy,bny->bnx", G, a["translation"]) + u, atol=1e-9)


def test_masked_rows_keep_s():
    inp = layer_inputs(7)
    out = ipa_layer(inp, DIMS)
    dead = ~inp["mask"]
    np.testing.assert_array_equal(out["s"][dead], inp["s"][dead])
