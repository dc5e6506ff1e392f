"""The CUDA path (through the C ABI) on cases with closed-form answers.

- The worked example of the BioTorch page "Invariant point attention (IPA)"
  ("Nearby frames receive more weight", eps = 1), in the factorised form
  (z1 = the printed pair values, z2 = identity, Wb = 0), with the printed w_out
  and with w_out picking the point-length feature, so that eps, which the page
  uses only inside the output point-length square root, changes the update.
- The pair-bias term alone (logit bullet of "Required behavior": pair_bias /
  sqrt(3)), two residues and two heads.
- A random bfloat16 batch with eps = 1 and w_out non-zero only on the length
  block: dropping eps, or adding it anywhere else, moves the update by more
  than the tolerance.

Each result is compared with the fp64 oracle at the stated tolerances, and the
worked example and the pair-bias case also with their closed forms."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import TOL, attach_structural, compare, to_device

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def handles():
    from protein_structure_models_b200 import Fipa, build
    build.build()
    h = {"f32": Fipa("f32", 0), "bf16": Fipa("bf16", 0)}
    yield h
    for x in h.values():
        x.close()


def _run(handles, inp, dtype):
    dev = to_device(inp, dtype)
    h = handles[dtype]
    out = h.forward(dev, eps=inp["eps"], want_attention=True, want_lse=True)
    h.sync_status()
    torch.cuda.synchronize()
    return out


def _sigmoid(x):
    return 1.0 / (1.0 + math.exp(-x))


def _worked_example(d, length_column):
    with open(os.path.join(GOLDEN, "worked_example_nearby_frames.json")) as f:
        pr = json.load(f)["printed_on_page"]
    pv = np.array(pr["pair_values_query_key"], float)          # [query, key]
    w_out = np.array(pr["w_out"], float)
    if length_column:
        w_out = np.array([[0.0], [0.0], [0.0], [0.0], [1.0], [0.0]])
    inp = dict(q=np.zeros((1, 2, 1, 1)), k=np.zeros((1, 2, 1, 1)),
               v=np.array(pr["v"], float).reshape(1, 2, 1, 1),
               q_points=np.zeros((1, 2, 1, 1, 3)), k_points=np.zeros((1, 2, 1, 1, 3)),
               v_points=np.tile(np.array([1.0, 0, 0]), (1, 2, 1, 1, 1)),
               rotation=np.tile(np.eye(3), (1, 2, 1, 1)),
               translation=np.array([[[0.0, 0, 0], [d, 0, 0]]]),
               z1=pv.reshape(1, 2, 2, 1), z2=np.eye(2).reshape(1, 2, 2, 1), Wb=np.zeros((1, 1)),
               point_weight_raw=np.zeros(1), w_out=w_out, b_out=np.array(pr["b_out"], float),
               mask=np.ones((1, 2), bool), pair_mask=None, eps=float(pr["eps"]))
    # closed form: L_00 = L_11 = 0, L_01 = L_10 = -c d^2, c = 1/2 ln2 sqrt(2/27)
    c = 0.5 * math.log(2.0) * math.sqrt(2.0 / 27.0)
    a_self = _sigmoid(c * d * d)
    a_other = 1.0 - a_self
    loc_x = [1.0 + a_other * d, 1.0 - a_other * d]
    if length_column:
        upd = [math.sqrt(x * x + inp["eps"]) for x in loc_x]
    else:
        upd = [3 * a_self + 9 * a_other, 6 * a_other + 8 * a_self]
    return inp, a_self, upd, loc_x


@pytest.mark.parametrize("length_column", [False, True], ids=["printed-w_out", "length-w_out"])
@pytest.mark.parametrize("d", [1.0, 3.0, 6.0])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_worked_example_eps1(handles, dtype, d, length_column):
    inp, a_self, upd, loc_x = _worked_example(d, length_column)
    assert inp["eps"] == 1.0
    out = _run(handles, inp, dtype)
    ref = oracle.ipa_forward_dense(inp, want_attention=True)
    attach_structural(ref, inp)
    compare(out, ref, dtype)
    tol = TOL[dtype]
    att = out["attention"].double().cpu().numpy()[0, 0]
    assert abs(att[0, 0] - a_self) <= tol["attention"] and abs(att[1, 1] - a_self) <= tol["attention"]
    assert att[0, 0] > att[0, 1] and att[1, 1] > att[1, 0]          # nearby frames get more weight
    u = out["update"].double().cpu().numpy()[0, :, 0]
    np.testing.assert_allclose(u, upd, atol=tol["update"], rtol=0)
    lp = out["local_points"].double().cpu().numpy()[0, :, 0, 0]
    np.testing.assert_allclose(lp[:, 0], loc_x, atol=tol["local_points"], rtol=0)
    np.testing.assert_allclose(lp[:, 1:], 0.0, atol=tol["local_points"], rtol=0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pair_bias_closed_form(handles, dtype):
    with open(os.path.join(GOLDEN, "pair_bias_two_residues.json")) as f:
        fx = json.load(f)
    H, Dv, Q, Cz = fx["H"], fx["Dv"], fx["Q"], fx["Cz"]
    F = H * (Dv + 4 * Q + Cz)
    inp = dict(q=np.zeros((1, 2, H, 1)), k=np.zeros((1, 2, H, 1)), v=np.ones((1, 2, H, Dv)),
               q_points=np.zeros((1, 2, H, 1, 3)), k_points=np.zeros((1, 2, H, 1, 3)),
               v_points=np.zeros((1, 2, H, Q, 3)), rotation=np.tile(np.eye(3), (1, 2, 1, 1)),
               translation=np.zeros((1, 2, 3)), z1=np.array(fx["z1_i_r_c"], float)[None],
               z2=np.array(fx["z2_j_r_c"], float)[None], Wb=np.array(fx["Wb_c_h"], float),
               point_weight_raw=np.zeros(H), w_out=np.eye(F), b_out=np.zeros(F),
               mask=np.ones((1, 2), bool), pair_mask=None, eps=1e-8)
    out = _run(handles, inp, dtype)
    ref = oracle.ipa_forward_dense(inp, want_attention=True)
    attach_structural(ref, inp)
    compare(out, ref, dtype)
    s3 = math.sqrt(3.0)
    a = {(0, 0): _sigmoid(3 / s3), (1, 0): _sigmoid(1 / s3), (0, 1): _sigmoid(1 / s3), (1, 1): _sigmoid(4 / s3)}
    att = out["attention"].double().cpu().numpy()[0]
    for (h, i), val in a.items():
        assert abs(att[h, i, i] - val) <= TOL[dtype]["attention"], (h, i, att[h, i, i], val)
    feat = out["update"].double().cpu().numpy()[0][:, 10:14]
    want = np.array([[a[0, 0], 0.0, a[1, 0], 0.0], [0.0, 2 * a[0, 1], 0.0, 2 * a[1, 1]]])
    np.testing.assert_allclose(feat, want, atol=TOL[dtype]["update"], rtol=0)


def test_random_batch_eps1_length_block(handles):
    """bf16 protein batch (2 samples of the protein-batch workload) with eps = 1
    and w_out zero outside the point-length block (scaled so the lengths carry
    the update).  sqrt(|x|^2 + 1) differs from sqrt(|x|^2 + 1e-8) by more than
    the 2e-2 tolerance for every |x| below ~25, so eps is exercised."""
    wl = workloads.workload(1).with_(B=2)
    inp = workloads.make_inputs(wl)
    inp["eps"] = 1.0
    H, Dv, Q = wl.H, wl.Dv, wl.Q
    lo, hi = H * Dv + 3 * H * Q, H * Dv + 4 * H * Q
    w = np.zeros_like(inp["w_out"])
    rng = np.random.default_rng(41)
    w[lo:hi] = workloads.round_to_dtype(rng.standard_normal((hi - lo, wl.Cout)) / math.sqrt(hi - lo), "bf16")
    inp["w_out"] = w
    out = _run(handles, inp, "bf16")
    ref = oracle.ipa_forward_dense(inp, want_attention=True)
    attach_structural(ref, inp)
    compare(out, ref, "bf16")
    # the same inputs with eps = 1e-8 give a clearly different update
    small = dict(inp, eps=1e-8)
    ref_small = oracle.ipa_forward_dense(small)
    assert np.max(np.abs(ref_small["update"] - ref["update"])) > 10 * TOL["bf16"]["update"]
