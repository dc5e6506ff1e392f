"""The IPA layer (fipa_ipa_layer, float32, through the C ABI) against the
layer oracle (oracle/layer.py): projection, core, residual and frame update.
Tolerance: the core's float32 bound, max-abs 1e-4, on s', local points, the
new rotations and the new translations."""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle.layer import ipa_layer, layer_widths

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module")
def handle():
    from protein_structure_models_b200 import Fipa, build
    build.build()
    h = Fipa("f32", 0)
    yield h
    h.close()


def make(seed, B, N, Cs, dims, walk=3.8, lengths=None, pair_mask=False):
    rng = np.random.default_rng(seed)
    H, Dv, Q, Cz = dims["H"], dims["Dv"], dims["Q"], dims["Cz"]
    _, Din = layer_widths(**dims)
    F = H * (Dv + 4 * Q + Cz)
    g = rng.standard_normal
    f32 = lambda x: np.asarray(x, np.float32).astype(np.float64)
    steps = g((B, N, 3))
    steps /= np.linalg.norm(steps, axis=-1, keepdims=True)
    steps[:, 0] = 0
    mask = np.ones((B, N), bool)
    if lengths is not None:
        mask = np.arange(N)[None, :] < rng.integers(lengths[0], lengths[1] + 1, size=B)[:, None]
    inp = dict(s=f32(g((B, N, Cs))), W_in=f32(g((Cs, Din)) / math.sqrt(Cs)), b_in=f32(0.1 * g(Din)),
               rotation=f32(workloads.random_rotations(rng, (B, N))), translation=f32(np.cumsum(walk * steps, 1)),
               mask=mask, pair_mask=None, Wb=f32(g((Cz, H))), point_weight_raw=f32(g(H)),
               w_out=f32(g((F, Cs)) / math.sqrt(F)), b_out=f32(g(Cs)), W_bb=f32(0.1 * g((Cs, 6)) / math.sqrt(Cs)),
               b_bb=f32(0.1 * g(6)), eps=1e-8)
    if pair_mask:
        pm = rng.random((B, N, N)) < 0.7
        pm[0, 2, :] = False
        inp["pair_mask"] = pm
    return inp


def check(handle, inp, dims):
    dev = {k: (torch.from_numpy(np.ascontiguousarray(v)).float().cuda() if isinstance(v, np.ndarray) and v.dtype != bool
               else (torch.from_numpy(np.ascontiguousarray(v)).cuda() if isinstance(v, np.ndarray) else v))
           for k, v in inp.items()}
    out = handle.ipa_layer(dev, dims, eps=inp["eps"])
    handle.sync_status()
    torch.cuda.synchronize()
    ref = ipa_layer(inp, dims)
    errs = {}
    for key in ("s", "rotation", "translation", "local_points"):
        got = out[key].double().cpu().numpy()
        errs[key] = float(np.max(np.abs(got - ref[key])))
    print(errs)
    assert all(v <= TOL for v in errs.values()), errs


def test_layer_small_with_masks(handle):
    dims = dict(H=2, D=4, Dv=4, P=2, Q=2, Cz=4, R=2)
    check(handle, make(1, 2, 40, 32, dims, lengths=(25, 40), pair_mask=True), dims)


def test_layer_protein_widths(handle):
    """Protein-batch widths (H=8, D=16, P=4, Q=8) with Cz=32, two ragged samples."""
    dims = dict(H=8, D=16, Dv=16, P=4, Q=8, Cz=32, R=2)
    check(handle, make(2, 2, 256, 64, dims, lengths=(60, 256)), dims)


def test_layer_rejects_bf16_handle():
    from protein_structure_models_b200 import Fipa
    from protein_structure_models_b200.fipa import FipaError
    h = Fipa("bf16", 0)
    try:
        dims = dict(H=2, D=4, Dv=4, P=2, Q=2, Cz=4, R=2)
        inp = make(3, 1, 8, 16, dims)
        dev = {k: (torch.from_numpy(np.ascontiguousarray(v)).float().cuda() if isinstance(v, np.ndarray) and v.dtype != bool
                   else (torch.from_numpy(np.ascontiguousarray(v)).cuda() if isinstance(v, np.ndarray) else v))
               for k, v in inp.items()}
        with pytest.raises(FipaError, match="UNSUPPORTED"):
            h.ipa_layer(dev, dims, workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
    finally:
        h.close()
