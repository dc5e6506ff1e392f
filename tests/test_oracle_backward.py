"""Pins of the fp64 backward oracle (oracle/backward.py) against what does not
share its code: central differences of the NumPy forward oracle, closed forms
and the invariances the page states ("Invariant point attention (IPA)",
Required behavior: the outputs are invariant under a global rigid motion)."""
import numpy as np
import pytest

import oracle
import workloads
from oracle import backward as bw


def _tiny(seed=5):
    wl = workloads.Workload("tiny-grad", 9, B=2, N=6, H=2, D=3, Dv=2, P=2, Q=2, Cz=3, R=2, Cout=4,
                            dtype="f32", frames="walk", t_scale=3.8)
    inp = workloads.make_inputs(wl, seed=seed)
    inp["mask"] = np.ones((2, 6), dtype=bool)
    inp["mask"][1, 5] = False                       # a masked residue (query and key)
    pm = np.ones((2, 6, 6), dtype=bool)
    pm[0, 2, :] = False                             # an empty neighbourhood
    pm[1, 0, 3] = False                             # one blocked pair
    inp["pair_mask"] = pm
    return inp


def _cotangents(inp, seed=11):
    rng = np.random.default_rng(seed)
    B, N, H = inp["q"].shape[:3]
    Q, Cout = inp["v_points"].shape[3], inp["w_out"].shape[1]
    return rng.standard_normal((B, N, Cout)), rng.standard_normal((B, N, H, Q, 3))


def _objective(inp, du, dl):
    out = oracle.ipa_forward_dense(inp)
    return float(np.sum(du * out["update"]) + np.sum(dl * out["local_points"]))


def test_restated_forward_matches_numpy_oracle():
    inp = _tiny()
    ref = oracle.ipa_forward_dense(inp)
    got = bw.forward(inp)
    assert np.max(np.abs(got["update"] - ref["update"])) < 1e-11
    assert np.max(np.abs(got["local_points"] - ref["local_points"])) < 1e-11


@pytest.mark.parametrize("key", bw.FLOAT_KEYS)
def test_vjp_matches_central_differences_of_numpy_oracle(key):
    """<grad_x f, delta> against (f(x + h delta) - f(x - h delta)) / 2h, f the
    NumPy oracle's <d_update, update> + <d_local, local_points>."""
    inp = _tiny()
    du, dl = _cotangents(inp)
    g = bw.ipa_vjp(inp, du, dl, wrt=[key])[key]
    rng = np.random.default_rng(100 + bw.FLOAT_KEYS.index(key))
    x0 = np.asarray(inp[key], np.float64)
    delta = rng.standard_normal(x0.shape)
    h = 1e-6 * max(1.0, float(np.max(np.abs(x0))))
    plus, minus = dict(inp), dict(inp)
    plus[key], minus[key] = x0 + h * delta, x0 - h * delta
    fd = (_objective(plus, du, dl) - _objective(minus, du, dl)) / (2 * h)
    an = float(np.sum(g * delta))
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (key, fd, an)


def test_bias_gradient_closed_form():
    """update = features w_out + b_out on rows with a non-empty neighbourhood,
    0 elsewhere: d f / d b_out = sum of d_update over those rows."""
    inp = _tiny()
    du, dl = _cotangents(inp)
    g = bw.ipa_vjp(inp, du, dl, wrt=["b_out"])["b_out"]
    mask, pm = inp["mask"], inp["pair_mask"]
    permitted = mask[:, :, None] & mask[:, None, :] & pm
    live = permitted.any(axis=2)
    assert np.allclose(g, du[live].sum(axis=0), atol=1e-12, rtol=0)


def test_empty_rows_carry_no_gradient():
    """Changing the cotangent of a row with an empty neighbourhood changes no
    gradient (its outputs are constant zeros)."""
    inp = _tiny()
    du, dl = _cotangents(inp)
    g0 = bw.ipa_vjp(inp, du, dl)
    du2, dl2 = du.copy(), dl.copy()
    du2[0, 2] += 5.0
    dl2[0, 2] -= 3.0
    g1 = bw.ipa_vjp(inp, du2, dl2)
    for key in bw.FLOAT_KEYS:
        assert np.allclose(g0[key], g1[key], atol=1e-12, rtol=0), key


def test_translation_gradients_sum_to_zero():
    """A common shift of every translation leaves the outputs unchanged, so the
    translation gradients of each sample sum to zero."""
    inp = _tiny()
    du, dl = _cotangents(inp)
    g = bw.ipa_vjp(inp, du, dl, wrt=["translation"])["translation"]
    scale = np.max(np.abs(g))
    assert scale > 1e-3
    assert np.max(np.abs(g.sum(axis=1))) < 1e-10 * max(1.0, scale)


def test_rotation_generator_is_a_null_direction():
    """Frames (R_i, t_i) -> (G R_i, G t_i) for a global rotation G leave the
    outputs unchanged; for G = exp(eps A), A antisymmetric, the first-order
    change sum_i <dR_i, A R_i> + <dt_i, A t_i> must vanish."""
    inp = _tiny()
    du, dl = _cotangents(inp)
    g = bw.ipa_vjp(inp, du, dl, wrt=["rotation", "translation"])
    R = np.asarray(inp["rotation"], np.float64)
    t = np.asarray(inp["translation"], np.float64)
    rng = np.random.default_rng(3)
    for _ in range(3):
        M = rng.standard_normal((3, 3))
        A = M - M.T
        for b in range(R.shape[0]):
            d = (np.sum(g["rotation"][b] * np.einsum("xy,nyz->nxz", A, R[b]))
                 + np.sum(g["translation"][b] * np.einsum("xy,ny->nx", A, t[b])))
            scale = np.max(np.abs(g["rotation"][b])) + np.max(np.abs(g["translation"][b]))
            assert abs(d) < 1e-9 * max(1.0, scale), d
