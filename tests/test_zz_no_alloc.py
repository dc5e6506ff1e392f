"""The allocation-free entry point, fipa_forward_noalloc, called through the C ABI.

Some callers of this library cannot allocate device memory where they run the
forward: a plugin inside a framework that owns every device allocation through
its own pool, or a latency-bound caller that may not call cudaMalloc mid-step.
fipa_forward_noalloc serves them with a fixed scratch array inside the library
instead of a caller-allocated workspace and a handle.

Checked here, on calls in a row that change shape and dtype in between (so
stale scratch from the previous call cannot stand in for this call's work):
every result matches the fp64 oracle at the parity tolerances and equals
fipa_forward's result bit for bit (same kernels, same launch order).

It sits in a file of its own, named to be collected last, and must pass both
alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import compare, to_device

pytestmark = pytest.mark.gpu


def _case(name):
    if name == "tiny-f32":
        return "f32", workloads.make_inputs(workloads.workload(0))
    if name == "protein-bf16":
        return "bf16", workloads.make_inputs(workloads.workload(1).with_(B=2))
    # ragged bf16: odd sizes, random masks, an empty neighbourhood and a fully masked sample
    wl = workloads.Workload("edge", 9, B=2, N=129, H=3, D=5, Dv=3, P=3, Q=5, Cz=7, R=3, Cout=20,
                            dtype="bf16", frames="walk", t_scale=3.8)
    inp = workloads.make_inputs(wl, seed=77)
    rng = np.random.default_rng(77)
    inp["mask"] = rng.random((2, 129)) < 0.7
    inp["mask"][1, :] = False
    pm = rng.random((2, 129, 129)) < 0.6
    pm[0, 4, :] = False
    inp["pair_mask"] = pm
    return "bf16", inp


def _noalloc(dev, inp, like):
    from protein_structure_models_b200.fipa import forward_noalloc
    o = {k: torch.full_like(like[k], float("nan")) for k in ("update", "local_points", "lse")}
    forward_noalloc(dev, eps=inp["eps"], out=o)
    torch.cuda.synchronize()
    return o


def test_noalloc_matches_oracle_and_forward():
    from protein_structure_models_b200 import Fipa, build
    build.build()
    names = ["protein-bf16", "tiny-f32", "ragged-bf16", "protein-bf16", "ragged-bf16", "tiny-f32"]
    cases = {n: _case(n) for n in set(names)}
    refs, fwd, handles = {}, {}, {}
    for n, (dtype, inp) in cases.items():
        refs[n] = oracle.ipa_forward_dense(inp)
        if dtype not in handles:
            handles[dtype] = Fipa(dtype, 0)
        h = handles[dtype]
        assert h.workspace_size(h.dims_of(inp)) <= 32 << 20
        dev = to_device(inp, dtype)
        fwd[n] = (dev, h.forward(dev, eps=inp["eps"], want_lse=True))
        h.sync_status()
    torch.cuda.synchronize()
    for n in names:
        dtype, inp = cases[n]
        dev, ref_gpu = fwd[n]
        o = _noalloc(dev, inp, ref_gpu)
        errs = compare(o, refs[n], dtype)
        print(n, errs)
        for k in ("update", "local_points", "lse"):
            assert torch.equal(torch.nan_to_num(o[k], nan=7.0), torch.nan_to_num(ref_gpu[k], nan=7.0)), (n, k)
    for h in handles.values():
        h.close()


def test_noalloc_rejects_oversized_problem():
    from protein_structure_models_b200 import build
    from protein_structure_models_b200.fipa import FipaError, forward_noalloc
    build.build()
    wl = workloads.workload("3-4096")           # ~70 MB of scratch: beyond the 32 MiB array
    inp = workloads.make_inputs(wl)
    dev = to_device(inp, "bf16")
    with pytest.raises(FipaError, match="WORKSPACE"):
        forward_noalloc(dev, eps=inp["eps"])


def test_noalloc_rejects_host_pointers():
    """Inputs that are not memory of the current device are refused before
    anything is launched."""
    from protein_structure_models_b200 import build
    from protein_structure_models_b200.fipa import INPUT_KEYS, make_dims, load_library
    build.build()
    lib = load_library()
    dtype, inp = _case("tiny-f32")
    host = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).float() for k in INPUT_KEYS + ("w_out", "b_out")}
    mask = torch.from_numpy(inp["mask"].astype(np.uint8))
    upd = torch.empty((1, 32, 32))
    lp = torch.empty((1, 32, 4, 8, 3))
    d = make_dims(**workloads.workload(0).dims())
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.fipa_forward_noalloc(0, *[p(host[k]) for k in INPUT_KEYS], p(mask), None, p(host["w_out"]),
                                  p(host["b_out"]), 1e-8, ctypes.byref(d), p(upd), p(lp), None, None)
    assert st == 1       # FIPA_ERR_INVALID_ARG
