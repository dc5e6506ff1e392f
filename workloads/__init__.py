"""Seeded synthetic inputs for the IPA aggregation core.

This module is shared by the oracle's tests, the CUDA parity tests and the
benchmark.  It holds only random draws and their shapes: no step of the
attention method itself is computed here.

The shapes and value families follow the five workloads of the IPA
aggregation core (page "Invariant point attention (IPA)", BioTorch, section
"Required behavior" for the tensor roles; FlashIPA, "Flash Invariant Point
Attention", for the factorised pair representation z_ij = z1_i^T z2_j with
factors of shape (B, L, r, d)).

Every value is drawn in float64 from a PCG64 generator and then rounded ONCE
to the workload's dtype (float32, or bfloat16 with round-to-nearest-even).
The rounded values are returned as float64 numpy arrays so that the oracle
and the GPU path consume bit-identical inputs.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "round_to_dtype",
           "random_rotations", "slice_batch", "SWEEP_N", "LONG_N", "BASE_SEED"]

BASE_SEED = 20261202
SWEEP_N = (512, 1024, 2048, 4096, 8192, 16384)
# lengths beyond the sweep, same recipe: the single-chain length that row
# sharding across GPUs exists for
LONG_N = (32768,)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Sizes and input recipe of one synthetic workload."""
    name: str
    index: int            # workload family number (0..4)
    B: int
    N: int
    H: int
    D: int
    Dv: int
    P: int
    Q: int
    Cz: int
    R: int
    Cout: int
    dtype: str            # "f32" or "bf16": dtype of every floating input
    frames: str           # "gauss" (t ~ N(0, t_scale^2)) or "walk" (random walk)
    t_scale: float        # std of translations ("gauss") or step length in Angstrom ("walk")
    len_range: Optional[tuple] = None   # per-sample valid length U{lo..hi}; None = all valid
    mask_p: Optional[float] = None      # Bernoulli keep-probability of residues (workload 0)
    empty_pair_row: bool = False        # one valid query whose pair_mask row is all False
    sweep_index: int = 0

    @property
    def F(self) -> int:
        return self.H * (self.Dv + 4 * self.Q + self.Cz)

    @property
    def seed(self) -> int:
        return BASE_SEED + 100 * self.index + self.sweep_index

    def dims(self) -> dict:
        return dict(B=self.B, N=self.N, H=self.H, D=self.D, Dv=self.Dv, P=self.P,
                    Q=self.Q, Cz=self.Cz, R=self.R, Cout=self.Cout)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _w0():
    return Workload("tiny-f32", 0, B=1, N=32, H=4, D=16, Dv=16, P=4, Q=8, Cz=8, R=2,
                    Cout=32, dtype="f32", frames="gauss", t_scale=10.0, mask_p=0.9,
                    empty_pair_row=True)


def _w1():
    return Workload("protein-batch-bf16", 1, B=8, N=256, H=8, D=16, Dv=16, P=4, Q=8,
                    Cz=128, R=2, Cout=256, dtype="bf16", frames="walk", t_scale=3.8,
                    len_range=(60, 256))


def _w2():
    return Workload("rna-chain-bf16", 2, B=1, N=2048, H=8, D=32, Dv=32, P=8, Q=8,
                    Cz=64, R=2, Cout=256, dtype="bf16", frames="walk", t_scale=6.0)


def _w3(n: int):
    return Workload(f"length-sweep-N{n}", 3, B=1, N=n, H=8, D=16, Dv=16, P=4, Q=8,
                    Cz=128, R=2, Cout=256, dtype="bf16", frames="walk", t_scale=3.8,
                    sweep_index=(SWEEP_N + LONG_N).index(n))


def _w4():
    return Workload("short-chain-batch-bf16", 4, B=512, N=150, H=8, D=16, Dv=16, P=4,
                    Q=8, Cz=64, R=2, Cout=256, dtype="bf16", frames="walk",
                    t_scale=6.0, len_range=(40, 150))


WORKLOADS = {"0": _w0(), "1": _w1(), "2": _w2(), "4": _w4()}
for _n in SWEEP_N + LONG_N:
    WORKLOADS[f"3-{_n}"] = _w3(_n)


def workload(key) -> Workload:
    """Look a workload up by key: 0, 1, 2, 4, or "3-<N>" for the length sweep."""
    return WORKLOADS[str(key)]


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values once to `dtype` and return them as float64.

    bf16 uses torch's round-to-nearest-even conversion; f32 uses numpy's."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        import torch
        t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)
        return t.to(torch.float64).numpy()
    raise ValueError(f"unknown dtype {dtype!r}")


def random_rotations(rng: np.random.Generator, shape) -> np.ndarray:
    """Proper rotation matrices from normalised N(0,1)^4 quaternions (w,x,y,z).

    Returns float64 [..., 3, 3], column-vector convention (x_global = R @ x)."""
    qv = rng.standard_normal(tuple(shape) + (4,))
    qv /= np.linalg.norm(qv, axis=-1, keepdims=True)
    w, x, y, z = (qv[..., i] for i in range(4))
    R = np.empty(tuple(shape) + (3, 3))
    R[..., 0, 0] = 1 - 2 * (y * y + z * z)
    R[..., 0, 1] = 2 * (x * y - w * z)
    R[..., 0, 2] = 2 * (x * z + w * y)
    R[..., 1, 0] = 2 * (x * y + w * z)
    R[..., 1, 1] = 1 - 2 * (x * x + z * z)
    R[..., 1, 2] = 2 * (y * z - w * x)
    R[..., 2, 0] = 2 * (x * z - w * y)
    R[..., 2, 1] = 2 * (y * z + w * x)
    R[..., 2, 2] = 1 - 2 * (x * x + y * y)
    return R


def _translations(rng, wl: Workload) -> np.ndarray:
    B, N = wl.B, wl.N
    if wl.frames == "gauss":
        return wl.t_scale * rng.standard_normal((B, N, 3))
    if wl.frames == "walk":
        u = rng.standard_normal((B, N, 3))
        u /= np.linalg.norm(u, axis=-1, keepdims=True)
        steps = wl.t_scale * u
        steps[:, 0, :] = 0.0            # t_0 = 0, t_{k+1} = t_k + s * u_k
        return np.cumsum(steps, axis=1)
    raise ValueError(wl.frames)


def make_inputs(wl: Workload, seed: Optional[int] = None) -> dict:
    """Draw one seeded input set for workload `wl`.

    Returns a dict of float64 numpy arrays already rounded to wl.dtype, plus
    bool masks.  Keys and layouts (row-major):
      q [B,N,H,D], k [B,N,H,D], v [B,N,H,Dv],
      q_points [B,N,H,P,3], k_points [B,N,H,P,3], v_points [B,N,H,Q,3],
      rotation [B,N,3,3], translation [B,N,3],
      z1 [B,N,R,Cz], z2 [B,N,R,Cz], Wb [Cz,H], point_weight_raw [H],
      mask [B,N] bool, pair_mask [B,N,N] bool or None,
      w_out [F,Cout], b_out [Cout], eps (float).
    """
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    B, N, H = wl.B, wl.N, wl.H
    g = rng.standard_normal
    raw = {
        "q": g((B, N, H, wl.D)),
        "k": g((B, N, H, wl.D)),
        "v": g((B, N, H, wl.Dv)),
        "q_points": g((B, N, H, wl.P, 3)),
        "k_points": g((B, N, H, wl.P, 3)),
        "v_points": g((B, N, H, wl.Q, 3)),
        "z1": g((B, N, wl.R, wl.Cz)),
        "z2": g((B, N, wl.R, wl.Cz)),
        "Wb": g((wl.Cz, H)),
        "point_weight_raw": g((H,)),
        "w_out": g((wl.F, wl.Cout)) / math.sqrt(wl.F),
        "b_out": g((wl.Cout,)),
    }
    raw["rotation"] = random_rotations(rng, (B, N))
    raw["translation"] = _translations(rng, wl)

    out = {key: round_to_dtype(val, wl.dtype) for key, val in raw.items()}

    if wl.len_range is not None:
        lo, hi = wl.len_range
        lengths = rng.integers(lo, hi + 1, size=B)
        mask = np.arange(N)[None, :] < lengths[:, None]
    elif wl.mask_p is not None:
        mask = rng.random((B, N)) < wl.mask_p
    else:
        mask = np.ones((B, N), dtype=bool)
    out["mask"] = mask

    pair_mask = None
    if wl.empty_pair_row:
        pair_mask = np.ones((B, N, N), dtype=bool)
        for b in range(B):
            valid = np.flatnonzero(mask[b])
            i_star = int(valid[rng.integers(0, len(valid))])
            pair_mask[b, i_star, :] = False
    out["pair_mask"] = pair_mask
    out["eps"] = 1e-8
    return out


_PER_SAMPLE = ("q", "k", "v", "q_points", "k_points", "v_points", "rotation", "translation",
               "z1", "z2", "mask")


def slice_batch(inp: dict, bsel) -> dict:
    """The inputs restricted to batch elements `bsel` (samples are independent)."""
    out = dict(inp)
    for key in _PER_SAMPLE:
        out[key] = inp[key][bsel]
    if inp.get("pair_mask") is not None:
        out["pair_mask"] = inp["pair_mask"][bsel]
    return out
