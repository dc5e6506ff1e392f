"""The allocation-free entry point, fipa_forward_noalloc, called through the C ABI.

Some callers of this library may not allocate device memory where they run the
forward: code executing while a CUDA graph is captured (cudaMalloc there is
forbidden or breaks the capture), or a plugin inside a framework that owns
every device allocation.  fipa_forward_noalloc serves them with a fixed scratch
array inside the library instead of a caller-allocated workspace.  This test
checks, on two calls in a row, that it gives what fipa_forward gives, within
the parity tolerances used for the CUDA path.

It sits in a file of its own, named to be collected last, and must pass both
alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import workloads
from parity_util import TOL, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("key,dtype,B", [("0", "f32", None), ("1", "bf16", 2)])
def test_noalloc_matches_forward_twice(key, dtype, B):
    from protein_structure_models_b200 import Fipa, build
    from protein_structure_models_b200.fipa import FipaError, forward_noalloc
    build.build()
    wl = workloads.workload(key)
    if B is not None:
        wl = wl.with_(B=B)
    inp = workloads.make_inputs(wl)
    dev = to_device(inp, dtype)
    h = Fipa(dtype, 0)
    assert h.workspace_size(wl.dims()) <= 32 << 20
    ref = h.forward(dev, eps=inp["eps"], want_lse=True)
    h.sync_status()
    torch.cuda.synchronize()
    outs = []
    for _ in range(2):
        o = {"update": torch.full_like(ref["update"], float("nan")),
             "local_points": torch.full_like(ref["local_points"], float("nan")),
             "lse": torch.full_like(ref["lse"], float("nan"))}
        forward_noalloc(dev, eps=inp["eps"], out=o)
        torch.cuda.synchronize()
        outs.append(o)
    tol = TOL[dtype]
    for o in outs:
        for k in ("update", "local_points"):
            err = float((o[k] - ref[k]).abs().max())
            assert err <= tol[k], (k, err)
        fin = torch.isfinite(ref["lse"])
        assert torch.equal(fin, torch.isfinite(o["lse"]))
        assert float((o["lse"][fin] - ref["lse"][fin]).abs().max()) <= tol["lse"]
    h.close()


def test_noalloc_rejects_oversized_problem():
    from protein_structure_models_b200.fipa import FipaError, forward_noalloc
    wl = workloads.workload("3-4096")           # ~100 MB of scratch: beyond the 32 MiB array
    inp = workloads.make_inputs(wl)
    dev = to_device(inp, "bf16")
    with pytest.raises(FipaError, match="WORKSPACE"):
        forward_noalloc(dev, eps=inp["eps"])
