"""Helpers shared by the GPU parity tests: device copies of the seeded inputs
and element-wise comparison with the oracle.

Tolerances: float32 inputs, max-abs 1e-4 on update, local_points and
attention; bfloat16 inputs, max-abs 2e-2 on update and local_points and 5e-3
on attention.  Structural zeros (not-permitted keys, empty neighbourhoods)
must be exactly zero.  The logsumexp output has no stated tolerance; it
carries the logit error directly, so it gets the logit-level bound
LSE_TOL (float32: 1e-3, bfloat16: 5e-2)."""
import numpy as np
import torch

TOL = {"f32": dict(update=1e-4, local_points=1e-4, attention=1e-4, lse=1e-3),
       "bf16": dict(update=2e-2, local_points=2e-2, attention=5e-3, lse=5e-2)}

FLOAT_KEYS = ("q", "k", "v", "q_points", "k_points", "v_points", "rotation", "translation",
              "z1", "z2", "Wb", "point_weight_raw", "w_out", "b_out")


def to_device(inp: dict, dtype: str, device="cuda") -> dict:
    """Exact device copies (the values are already rounded to `dtype`)."""
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(device=device, dtype=td) for k in FLOAT_KEYS}
    out["mask"] = torch.from_numpy(np.ascontiguousarray(inp["mask"])).to(device)
    pm = inp.get("pair_mask")
    out["pair_mask"] = None if pm is None else torch.from_numpy(np.ascontiguousarray(pm)).to(device)
    return out


from workloads import slice_batch  # noqa: E402,F401  (re-exported for the tests)


def max_err(a, b):
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def compare(gpu: dict, ref: dict, dtype: str, rows=None, bsel=None, check_attention=True):
    """Compare GPU outputs (full tensors) with oracle outputs computed for
    batch elements `bsel` (default all) and query rows `rows` (default all).
    Returns a dict of max-abs errors; raises AssertionError on a violation."""
    tol = TOL[dtype]
    g = {k: v.detach().double().cpu().numpy() for k, v in gpu.items() if v is not None}
    if bsel is not None:
        g = {k: v[bsel] for k, v in g.items()}
    if rows is not None:
        g["update"] = g["update"][:, rows]
        g["local_points"] = g["local_points"][:, rows]
        if "attention" in g:
            g["attention"] = g["attention"][:, :, rows]
        if "lse" in g:
            g["lse"] = g["lse"][:, :, rows]
    errs = {}
    empty = np.all(np.isneginf(ref["lse"]), axis=1)          # [B, rows]
    for key in ("update", "local_points"):
        errs[key] = max_err(g[key], ref[key])
        assert errs[key] <= tol[key], f"{key}: max-abs error {errs[key]:.3e} > {tol[key]}"
        assert np.all(g[key][empty] == 0.0), f"{key}: empty neighbourhood not exactly zero"
    if "lse" in g:
        fin = np.isfinite(ref["lse"])
        assert np.array_equal(fin, np.isfinite(g["lse"])), "lse: -inf pattern differs"
        errs["lse"] = max_err(g["lse"][fin], ref["lse"][fin])
        assert errs["lse"] <= tol["lse"], f"lse: max-abs error {errs['lse']:.3e}"
    if check_attention and "attention" in g and "attention" in ref:
        zero = ref["attention"] == 0.0
        errs["attention"] = max_err(g["attention"], ref["attention"])
        assert errs["attention"] <= tol["attention"], f"attention: {errs['attention']:.3e}"
        # structural zeros are exact: every not-permitted entry must be 0 on the GPU
        structural = structural_zero_mask(ref)
        assert np.all(g["attention"][structural] == 0.0), "attention: structural zero violated"
        errs["attention_zero_frac"] = float(zero.mean())
    return errs


def structural_zero_mask(ref):
    return ref["_structural"] if "_structural" in ref else np.zeros_like(ref["attention"], dtype=bool)


def attach_structural(ref: dict, inp: dict, rows=None):
    """Mark entries that are zero by the mask rule (not by underflow)."""
    mask = inp["mask"].astype(bool)
    B, N = mask.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    pm = inp.get("pair_mask")
    permitted = mask[:, rows, None] & mask[:, None, :]
    if pm is not None:
        permitted = permitted & pm[:, rows, :]
    empty = ~permitted.any(-1)
    structural = ~permitted | empty[..., None]
    H = ref["attention"].shape[1]
    ref["_structural"] = np.broadcast_to(structural[:, None], (B, H, len(rows), N))
    return ref
