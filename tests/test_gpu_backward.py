"""The CUDA backward pass (fipa_backward, through the C ABI) against the fp64
backward oracle (oracle/backward.py: the vector-Jacobian product of the page's
forward, "Invariant point attention (IPA)", Required behavior; the page's
"Starter code" section grades the suite "including gradients").

Tolerance (fp16 products for bfloat16 and float32 inputs alike): for every
gradient tensor, max |g - g_ref| <= GRAD_TOL * max |g_ref|, GRAD_TOL = 1e-2.
The fp16 operands of the recomputed products and of dS carry 2^-11 relative
rounding each; dS = P (dP - D) loses up to a few bits where dP is close to D;
1e-2 allows a 20x amplification of one fp16 rounding.  Residues with mask 0
pass no gradient at all, so theirs must be exactly zero."""
import numpy as np
import pytest
import torch

import workloads
from oracle import backward as bw
from parity_util import to_device

pytestmark = pytest.mark.gpu

GRAD_TOL = 1e-2


@pytest.fixture(scope="module")
def handle():
    from protein_structure_models_b200 import Fipa, build
    build.build()
    h = Fipa("bf16", 0)
    yield h
    h.close()


def _cotangents(inp, seed):
    rng = np.random.default_rng(seed)
    B, N, H = inp["q"].shape[:3]
    Q, Cout = inp["v_points"].shape[3], inp["w_out"].shape[1]
    return rng.standard_normal((B, N, Cout)), rng.standard_normal((B, N, H, Q, 3))


def run_backward(handle, inp, du, dl):
    dev = to_device(inp, "bf16")
    d_update = torch.from_numpy(du).float().cuda().contiguous()
    d_local = torch.from_numpy(dl).float().cuda().contiguous()
    g = handle.backward(dev, d_update, d_local, eps=inp["eps"])
    handle.sync_status()
    torch.cuda.synchronize()
    return {k: v.double().cpu().numpy() for k, v in g.items()}


def check_grads(handle, inp, seed=3):
    du, dl = _cotangents(inp, seed)
    got = run_backward(handle, inp, du, dl)
    ref = bw.ipa_vjp(inp, du, dl)
    errs = {}
    for key in bw.FLOAT_KEYS:
        scale = float(np.max(np.abs(ref[key])))
        err = float(np.max(np.abs(got[key] - ref[key])))
        errs[key] = err / scale if scale > 0 else err
    print({k: f"{v:.2e}" for k, v in errs.items()})
    bad = {k: v for k, v in errs.items() if v > GRAD_TOL}
    assert not bad, bad
    # masked residues pass no gradient back
    dead = ~np.asarray(inp["mask"]).astype(bool)
    if dead.any():
        for key in ("q", "k", "v", "q_points", "k_points", "v_points", "rotation", "translation", "z1", "z2"):
            assert np.all(got[key][dead] == 0.0), key
    return errs


def _custom(seed, **kw):
    base = dict(B=2, N=40, H=3, D=5, Dv=3, P=3, Q=5, Cz=7, R=3, Cout=20)
    base.update(kw)
    wl = workloads.Workload("edge", 9, dtype="bf16", frames="walk", t_scale=3.8, **base)
    return workloads.make_inputs(wl, seed=seed)


def test_backward_small_masks_and_empty_rows(handle):
    inp = _custom(7, N=40)
    rng = np.random.default_rng(7)
    inp["mask"] = rng.random(inp["mask"].shape) < 0.8
    inp["mask"][1, 30:] = False
    pm = rng.random((2, 40, 40)) < 0.7
    pm[0, 3, :] = False                                   # an empty neighbourhood
    inp["pair_mask"] = pm
    check_grads(handle, inp)


def test_backward_masked_tiles_and_pair_mask(handle):
    """Fully masked query and key tiles between valid ones (the forward's early
    exit, the k side's zeroed rows) and a pair mask over a ragged last tile
    (N = 300: the mask bits past N)."""
    inp = _custom(23, N=384)
    rng = np.random.default_rng(23)
    m = rng.random((2, 384)) < 0.8
    m[0, 128:256] = False
    m[1, :128] = False
    inp["mask"] = m
    inp["pair_mask"] = rng.random((2, 384, 384)) < 0.7
    check_grads(handle, inp)
    inp = _custom(29, N=300, B=1)
    inp["pair_mask"] = rng.random((1, 300, 300)) < 0.5
    check_grads(handle, inp, seed=29)


@pytest.mark.parametrize("N", [1, 129, 300])
def test_backward_ragged_tiles(handle, N):
    inp = _custom(100 + N, N=N, B=1 if N == 300 else 2)
    check_grads(handle, inp, seed=N)


def test_backward_protein_batch(handle):
    """Two samples of the protein-batch workload (B=8, N=256, Cz=128), padded
    lengths masked."""
    inp = workloads.make_inputs(workloads.workload(1).with_(B=2))
    check_grads(handle, inp)


def test_backward_long_chain_multi_tile(handle):
    """Four query and key tiles of one chain (the length-sweep recipe, N=512)."""
    check_grads(handle, workloads.make_inputs(workloads.workload("3-512")))


def test_backward_rna_dims(handle):
    """The RNA-chain widths (D=32, P=8, Cz=64) on a 256-residue chain."""
    check_grads(handle, workloads.make_inputs(workloads.workload(2).with_(N=256)))


def test_backward_short_chain_batch(handle):
    """Four samples of the short-chain batch (N=150, lengths U{40..150})."""
    inp = workloads.make_inputs(workloads.workload(4).with_(B=4))
    check_grads(handle, inp)


RIGID_TOL = 1e-3


@pytest.mark.parametrize("key", ["1", "3-4096", "3-16384"])
def test_backward_rigid_motion_identities(handle, key):
    """Sizes the fp64 oracle cannot differentiate, checked by identities that
    hold at any size.  The outputs are unchanged when every frame of a sample
    takes the same rigid motion (page "Invariant point attention (IPA)",
    Required behavior: invariant features and local points), so per sample
    the translation gradients sum to zero, and for each rotation generator
    Omega, sum_i <dR_i, Omega R_i> + <dt_i, Omega t_i> = 0.  The computed sums
    carry the rounding of the fp16 products (2^-11 relative each), not aligned
    across residues: bound RIGID_TOL of the sum of the terms' magnitudes
    (about two roundings).  Measured: <= 4e-5 (protein batch), ~1e-6 (N = 4096,
    16384)."""
    inp = workloads.make_inputs(workloads.workload(key))
    du, dl = _cotangents(inp, 7)
    g = run_backward(handle, inp, du, dl)
    R = np.asarray(inp["rotation"], np.float64)
    t = np.asarray(inp["translation"], np.float64)
    gR, gt = g["rotation"], g["translation"]
    gens = []
    for i, j in ((1, 2), (2, 0), (0, 1)):
        om = np.zeros((3, 3))
        om[i, j], om[j, i] = -1.0, 1.0
        gens.append(om)
    for b in range(R.shape[0]):
        ratio_t = np.abs(gt[b].sum(0)) / np.abs(gt[b]).sum(0)
        assert np.all(ratio_t <= RIGID_TOL), (b, ratio_t)
        for om in gens:
            term_r = gR[b] * np.einsum("xy,nyz->nxz", om, R[b])
            term_t = gt[b] * np.einsum("xy,ny->nx", om, t[b])
            s = term_r.sum() + term_t.sum()
            scale = np.abs(term_r).sum() + np.abs(term_t).sum()
            assert abs(s) <= RIGID_TOL * scale, (b, s, scale)


def test_backward_deterministic(handle):
    inp = _custom(11, N=200)
    du, dl = _cotangents(inp, 5)
    a = run_backward(handle, inp, du, dl)
    b = run_backward(handle, inp, du, dl)
    for key in a:
        assert np.array_equal(a[key], b[key]), key


def test_backward_float32_inputs():
    """float32 inputs: the recompute reads them in the bfloat16 lifted layout
    (fp16 products), so the same 1e-2 normwise bound applies; the tiny float32
    workload (masks, an empty pair row) and an odd-width ragged case."""
    from protein_structure_models_b200 import Fipa
    h = Fipa("f32", 0)
    try:
        for inp in (workloads.make_inputs(workloads.workload(0)), _custom_f32(31, N=129)):
            du, dl = _cotangents(inp, 4)
            dev = to_device(inp, "f32")
            g = h.backward(dev, torch.from_numpy(du).float().cuda(), torch.from_numpy(dl).float().cuda(),
                           eps=inp["eps"])
            h.sync_status()
            torch.cuda.synchronize()
            got = {k: v.double().cpu().numpy() for k, v in g.items()}
            ref = bw.ipa_vjp(inp, du, dl)
            errs = {k: float(np.max(np.abs(got[k] - ref[k])) / max(1e-30, float(np.max(np.abs(ref[k])))))
                    for k in bw.FLOAT_KEYS}
            print({k: f"{v:.2e}" for k, v in errs.items()})
            assert all(v <= GRAD_TOL for v in errs.values()), errs
    finally:
        h.close()


def _custom_f32(seed, **kw):
    base = dict(B=2, N=40, H=3, D=5, Dv=3, P=3, Q=5, Cz=7, R=3, Cout=20)
    base.update(kw)
    wl = workloads.Workload("edge32", 9, dtype="f32", frames="walk", t_scale=3.8, **base)
    return workloads.make_inputs(wl, seed=seed)


def test_saved_backward_rejects_float32():
    from protein_structure_models_b200 import Fipa
    from protein_structure_models_b200.fipa import FipaError
    h = Fipa("f32", 0)
    try:
        inp = workloads.make_inputs(workloads.workload(0))
        dev = to_device(inp, "f32")
        du = torch.zeros((1, 32, 32), dtype=torch.float32, device="cuda")
        with pytest.raises(FipaError, match="UNSUPPORTED"):
            h.backward(dev, du, workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"), saved=True)
    finally:
        h.close()


def test_backward_stage_times(handle):
    """With stage timing on, fipa_backward records its five stages."""
    inp = _custom(13, N=129)
    du, dl = _cotangents(inp, 2)
    handle.enable_stage_timing(True)
    try:
        run_backward(handle, inp, du, dl)
        st = handle.backward_stage_times()
    finally:
        handle.enable_stage_timing(False)
    assert list(st) == ["recompute", "prep", "q_side", "k_side", "chain"]
    assert all(v > 0.0 for v in st.values()), st


def test_forward_train_and_saved_backward(handle):
    """fipa_forward_train gives fipa_forward's outputs, and fipa_backward_saved
    (no recompute) gives fipa_backward's gradients, both bit for bit."""
    inp = workloads.make_inputs(workloads.workload(1).with_(B=2))
    dev = to_device(inp, "bf16")
    du, dl = _cotangents(inp, 9)
    d_update = torch.from_numpy(du).float().cuda().contiguous()
    d_local = torch.from_numpy(dl).float().cuda().contiguous()
    ref_fwd = handle.forward(dev, eps=inp["eps"], want_lse=True)
    ref_bwd = handle.backward(dev, d_update, d_local, eps=inp["eps"])
    ws = torch.empty(handle.backward_workspace_size(handle.dims_of(dev)), dtype=torch.uint8, device="cuda")
    fwd = handle.forward_train(dev, ws, eps=inp["eps"], want_lse=True)
    bwd = handle.backward(dev, d_update, d_local, eps=inp["eps"], workspace=ws, saved=True)
    handle.sync_status()
    torch.cuda.synchronize()
    for k in ("update", "local_points", "lse"):
        assert torch.equal(torch.nan_to_num(fwd[k], nan=7.0), torch.nan_to_num(ref_fwd[k], nan=7.0)), k
    for k in ref_bwd:
        assert torch.equal(bwd[k], ref_bwd[k]), k


def test_backward_value_buffer_recompute(handle):
    """A 1024-residue chain (8 key tiles: the recompute's core runs in
    value-buffer mode) at reduced widths so the dense fp64 oracle stays small."""
    wl = workloads.Workload("grad-vb", 9, B=1, N=1024, H=2, D=16, Dv=16, P=4, Q=8, Cz=32, R=2, Cout=32,
                            dtype="bf16", frames="walk", t_scale=3.8)
    check_grads(handle, workloads.make_inputs(wl, seed=21))


def test_backward_single_half_pair_operand(monkeypatch):
    """FIPA_PAIR_SPLIT=0: the pair-bias operand as one fp16 half (the backward
    kernels' single-half branch)."""
    from protein_structure_models_b200 import Fipa
    monkeypatch.setenv("FIPA_PAIR_SPLIT", "0")
    h = Fipa("bf16", 0)
    try:
        check_grads(h, _custom(23, N=200))
    finally:
        h.close()
