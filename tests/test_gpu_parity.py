"""CUDA path vs the fp64 oracle on the same seeded inputs (needs a B200).

Every call goes through the C ABI (libfipa.so) via the ctypes binding."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import attach_structural, compare, slice_batch, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def handles():
    from protein_structure_models_b200 import Fipa, build
    build.build()
    h = {"f32": Fipa("f32", 0), "bf16": Fipa("bf16", 0)}
    yield h
    for x in h.values():
        x.close()


def run_gpu(handles, inp, dtype, want_attention=True):
    dev = to_device(inp, dtype)
    h = handles[dtype]
    out = h.forward(dev, eps=inp["eps"], want_attention=want_attention, want_lse=True)
    h.sync_status()
    torch.cuda.synchronize()
    return out


def check(handles, inp, dtype, rows=None, bsel=None, want_attention=True):
    gpu = run_gpu(handles, inp, dtype, want_attention)
    ref_inp = inp if bsel is None else slice_batch(inp, bsel)
    ref = oracle.ipa_forward_dense(ref_inp, rows=rows, want_attention=want_attention)
    if want_attention:
        attach_structural(ref, ref_inp, rows)
    errs = compare(gpu, ref, dtype, rows=rows, bsel=bsel, check_attention=want_attention)
    print(errs)
    return gpu, errs


# ------------------------------------------------------------------ the five workloads
def test_workload0_tiny_f32(handles):
    inp = workloads.make_inputs(workloads.workload(0))
    check(handles, inp, "f32")


def test_workload0_float32_long_chain(handles):
    """The float32 path on a long chain (N = 4096: 32 key tiles per query tile,
    the exact point term over every key group, O accumulated by the tensor
    cores in segments of a few key tiles and added in fp32 on the CUDA cores,
    normalised by its own sum of P), on sampled rows."""
    n = 4096
    inp = workloads.make_inputs(workloads.workload(0).with_(N=n))
    rng = np.random.default_rng(40)
    rows = np.unique(np.concatenate([[0, 127, 128, n - 1], rng.choice(n, 60, replace=False)]))
    check(handles, inp, "f32", rows=rows, want_attention=False)


def test_workload1_protein_batch(handles):
    inp = workloads.make_inputs(workloads.workload(1))
    check(handles, inp, "bf16")
    check(handles, inp, "bf16", want_attention=False)   # as the benchmark runs it


def test_workload2_rna_chain_sampled_rows(handles):
    inp = workloads.make_inputs(workloads.workload(2))
    rng = np.random.default_rng(2)
    rows = np.sort(np.concatenate([[0, 127, 128, 2047], rng.choice(2048, 124, replace=False)]))
    check(handles, inp, "bf16", rows=np.unique(rows))


@pytest.mark.parametrize("n", [512, 1024, 2048, 4096])
def test_workload3_length_sweep(handles, n):
    inp = workloads.make_inputs(workloads.workload(f"3-{n}"))
    rng = np.random.default_rng(n)
    rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 96, replace=False)]))
    check(handles, inp, "bf16", rows=rows, want_attention=(n <= 2048))


@pytest.mark.parametrize("n", [8192, 16384, 32768])
def test_workload3_long_chains(handles, n):
    inp = workloads.make_inputs(workloads.workload(f"3-{n}"))
    rng = np.random.default_rng(n)
    rows = np.unique(np.concatenate([[0, 128, n - 1], rng.choice(n, 45, replace=False)]))
    check(handles, inp, "bf16", rows=rows, want_attention=False)


def test_workload4_short_chain_batch(handles):
    inp = workloads.make_inputs(workloads.workload(4))
    bsel = np.arange(0, 512, 16)           # 32 of the 512 samples, checked in full
    check(handles, inp, "bf16", bsel=bsel)
    check(handles, inp, "bf16", bsel=bsel, want_attention=False)


# ------------------------------------------------------------------ edge cases
def _custom(dtype, seed, **kw):
    base = dict(B=2, N=40, H=3, D=5, Dv=3, P=3, Q=5, Cz=7, R=3, Cout=20)
    base.update(kw)
    wl = workloads.Workload("edge", 9, dtype=dtype, frames="walk", t_scale=3.8, len_range=None,
                            **base)
    inp = workloads.make_inputs(wl, seed=seed)
    return inp


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 2, 127, 129, 300])
def test_ragged_and_odd_sizes(handles, dtype, N):
    inp = _custom(dtype, 100 + N, N=N)
    check(handles, inp, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_masks_and_empty_rows(handles, dtype):
    inp = _custom(dtype, 7, N=200)
    rng = np.random.default_rng(7)
    inp["mask"] = rng.random(inp["mask"].shape) < 0.7
    inp["mask"][1, :] = False                                   # a fully masked sample
    pm = rng.random((2, 200, 200)) < 0.6
    pm[0, 5, :] = False                                          # empty neighbourhood
    pm[0, :, 130:] = False                                       # a whole key tile blocked
    inp["pair_mask"] = pm
    check(handles, inp, dtype)
    check(handles, inp, dtype, want_attention=False)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fully_masked_query_tiles(handles, dtype):
    """A query tile without a valid residue leaves the core at entry, writing
    only what an empty row gets (row statistics, lse -inf, zero local points,
    the row flag): a masked middle tile and a masked first tile between valid
    ones, with and without a pair mask."""
    inp = _custom(dtype, 21, N=384)
    rng = np.random.default_rng(21)
    m = rng.random((2, 384)) < 0.8
    m[0, 128:256] = False
    m[1, :128] = False
    inp["mask"] = m
    check(handles, inp, dtype)
    check(handles, inp, dtype, want_attention=False)
    inp["pair_mask"] = rng.random((2, 384, 384)) < 0.7
    check(handles, inp, dtype)


def test_single_head_single_point(handles):
    inp = _custom("bf16", 11, N=64, H=1, P=1, Q=1, D=1, Dv=1, Cz=1, R=1, Cout=1)
    check(handles, inp, "bf16")


def test_rigid_motion_invariance_on_gpu(handles):
    inp = workloads.make_inputs(workloads.workload(1))
    a = run_gpu(handles, inp, "bf16", want_attention=False)
    rng = np.random.default_rng(5)
    G = workloads.random_rotations(rng, ())
    moved = dict(inp)
    moved["rotation"] = workloads.round_to_dtype(np.einsum("xy,bnyz->bnxz", G, inp["rotation"]), "bf16")
    moved["translation"] = workloads.round_to_dtype(
        np.einsum("xy,bny->bnx", G, inp["translation"]) + 25.0, "bf16")
    b = run_gpu(handles, moved, "bf16", want_attention=False)
    # the moved frames are re-rounded to bf16, so compare each against its own oracle
    ref_b = oracle.ipa_forward_dense(moved, rows=np.arange(0, 256, 8))
    gb = b["update"].double().cpu().numpy()[:, ::8]
    assert np.max(np.abs(gb - ref_b["update"])) <= 2e-2
    assert torch.equal(a["update"].isfinite(), b["update"].isfinite())


def test_deterministic(handles):
    inp = workloads.make_inputs(workloads.workload(1))
    a = run_gpu(handles, inp, "bf16", want_attention=False)
    b = run_gpu(handles, inp, "bf16", want_attention=False)
    assert torch.equal(a["update"], b["update"])
    assert torch.equal(a["local_points"], b["local_points"])


# ------------------------------------------------------------------ host-side validation
def test_validation_errors(handles):
    from protein_structure_models_b200.fipa import FipaError
    inp = to_device(workloads.make_inputs(workloads.workload(0)), "f32")
    h = handles["f32"]
    bad = dict(inp)
    bad["q"] = inp["q"].to(torch.bfloat16)
    with pytest.raises(ValueError):
        h.forward(bad)
    with pytest.raises(FipaError, match="WORKSPACE"):
        h.forward(inp, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(FipaError, match="INVALID_ARG"):
        h.forward(inp, eps=-1.0)
    with pytest.raises(FipaError, match="INVALID_ARG"):
        h.workspace_size(dict(B=1, N=0, H=1, D=1, Dv=1, P=1, Q=1, Cz=1, R=1, Cout=1))
    with pytest.raises(FipaError, match="UNSUPPORTED"):
        h.workspace_size(dict(B=1, N=8, H=1, D=1, Dv=1, P=65, Q=1, Cz=1, R=1, Cout=1))
    h.sync_status()


# ------------------------------------------------------------------ core modes
@pytest.mark.parametrize("env", [{"FIPA_VALUE_BUFFER": "0"}, {"FIPA_VALUE_BUFFER": "2"}],
                         ids=["ring-only", "value-buffer"])
def test_core_modes(handles, monkeypatch, env):
    """The core's value-buffer mode (value chunks of each key tile in a buffer of
    their own) is chosen by sample length; force it off and on for short and
    long samples so both paths stay parity-checked at every size class."""
    from protein_structure_models_b200 import Fipa
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    h = {"bf16": Fipa("bf16", 0)}
    try:
        # without the attention output, as the benchmark runs it
        check(h, workloads.make_inputs(workloads.workload(1)), "bf16", want_attention=False)
        for n in (1, 2, 129, 300):
            check(h, _custom("bf16", 200 + n, N=n), "bf16", want_attention=False)
        n = 1024
        inp = workloads.make_inputs(workloads.workload(f"3-{n}"))
        rows = np.unique(np.concatenate([[0, 127, 128, n - 1], np.random.default_rng(7).choice(n, 60, replace=False)]))
        check(h, inp, "bf16", rows=rows, want_attention=False)
    finally:
        h["bf16"].close()


# ------------------------------------------------------------------ query-row ranges
def _row_range_case(handles, dtype, inp, world, want_attention=True):
    """fipa_forward_rows over the ranges of a `world`-way tile split (balanced by
    valid tiles, as a multi-GPU run shards one sample) must rebuild the full
    forward bit for bit; rows of no range stay untouched (NaN sentinel)."""
    from protein_structure_models_b200.sharding import tile_rows, tile_shards
    dev = to_device(inp, dtype)
    h = handles[dtype]
    wa = want_attention
    full = h.forward(dev, eps=inp["eps"], want_attention=wa, want_lse=True)
    B, N = inp["mask"].shape
    T = (N + 127) // 128
    weights = [int(inp["mask"][:, t * 128:(t + 1) * 128].any()) for t in range(T)]
    out = {k: torch.full_like(v, float("nan")) for k, v in full.items()}
    ranges = [tile_rows(r, N) for r in tile_shards(weights, world)]
    for r0, r1 in ranges:
        if r0 < r1:
            h.forward(dev, eps=inp["eps"], want_attention=wa, want_lse=True, out=out, rows=(r0, r1))
    h.sync_status()
    torch.cuda.synchronize()
    for k in full:
        assert torch.equal(torch.nan_to_num(out[k], nan=7.0), torch.nan_to_num(full[k], nan=7.0)), k
    # a single middle range: the rows outside it are not written
    if N > 256:
        part = {k: torch.full_like(v, float("nan")) for k, v in full.items()}
        h.forward(dev, eps=inp["eps"], want_attention=wa, want_lse=True, out=part, rows=(128, 256))
        torch.cuda.synchronize()
        for k, v in part.items():
            rows_axis = 2 if k in ("attention", "lse") else 1
            inside = v.narrow(rows_axis, 128, 128)
            assert torch.equal(inside, full[k].narrow(rows_axis, 128, 128)), k
            outside = torch.cat([v.narrow(rows_axis, 0, 128), v.narrow(rows_axis, 256, N - 256)], rows_axis)
            assert torch.isnan(outside).all(), k


def test_row_ranges_long_chain(handles):
    _row_range_case(handles, "bf16", workloads.make_inputs(workloads.workload("3-1024")), 3)


def test_row_ranges_32768_chain(handles):
    """The 32768-residue chain (beyond the length sweep; the length that row
    sharding across GPUs exists for) split 3 ways rebuilds the full forward bit
    for bit.  Its parity with the oracle is test_workload3_long_chains[32768]."""
    _row_range_case(handles, "bf16", workloads.make_inputs(workloads.workload("3-32768")), 3,
                    want_attention=False)


def test_row_ranges_ragged_batch(handles):
    inp = _custom("bf16", 31, B=3, N=300)
    inp["mask"][1, 200:] = False
    _row_range_case(handles, "bf16", inp, 2)


def test_row_ranges_f32(handles):
    _row_range_case(handles, "f32", _custom("f32", 32, N=300), 2)


def test_row_ranges_rejected(handles):
    from protein_structure_models_b200.fipa import FipaError
    inp = _custom("bf16", 33, N=300)
    dev = to_device(inp, "bf16")
    for rows in [(0, 0), (64, 256), (0, 200), (256, 128), (0, 301), (-128, 128)]:
        with pytest.raises(FipaError):
            handles["bf16"].forward(dev, eps=inp["eps"], rows=rows)
