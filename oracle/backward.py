"""fp64 gradients of the IPA aggregation core -- TEST INFRASTRUCTURE ONLY.

Same import rules as the `oracle` package: only `tests/`,
`__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` may use it;
it imports nothing from the product path.

The backward of the forward defined on the BioTorch page "Invariant point
attention (IPA)", section "Required behavior" (the reading of the pair
representation is that of `oracle.ipa_forward_dense`: z_ij = sum_r z1_ir z2_jr,
pair_bias_ijh = sum_c z_ij[c] Wb[c,h]).  The forward is restated here in
float64 PyTorch CPU ops, term for term as the page orders it, so that the
vector-Jacobian product

    grad_x <d_update, update(x)> + <d_local, local_points(x)>

is the exact derivative (up to rounding) for every floating input x.  Masks
are inputs, not variables.  Two details keep every gradient finite: the
softmax shift (the row maximum) is held constant, which leaves the value and
its derivative unchanged, and not-permitted logits enter the exponential as
zeros before they are masked out.

Pinned in tests/test_oracle_backward.py against what does not share this code:
central finite differences of the NumPy oracle `ipa_forward_dense` along
random directions for every input, the bias gradient in closed form,
translation and rotation invariance of the outputs (their infinitesimal forms
on the frame gradients), and the zero contribution of empty neighbourhoods.

Dense N x N x Cz pair tensors: small sizes only.
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, Optional

import numpy as np
import torch

FLOAT_KEYS = ("q", "k", "v", "q_points", "k_points", "v_points", "rotation", "translation",
              "z1", "z2", "Wb", "point_weight_raw", "w_out", "b_out")


def _softplus(x: torch.Tensor) -> torch.Tensor:
    """log(1 + e^x) = max(x, 0) + log1p(e^-|x|), without overflow."""
    return torch.clamp_min(x, 0.0) + torch.log1p(torch.exp(-torch.abs(x)))


def forward_torch(t: Dict[str, torch.Tensor], mask: torch.Tensor, pair_mask: torch.Tensor,
                  eps: float):
    """update [B,N,Cout] and local_points [B,N,H,Q,3] from float64 tensors `t`
    (keys FLOAT_KEYS, layouts as `workloads.make_inputs`), mask [B,N] and
    pair_mask [B,N,N] (bool)."""
    q, k, v = t["q"], t["k"], t["v"]
    rot, trans = t["rotation"], t["translation"]
    B, N, H, D = q.shape
    P = t["q_points"].shape[3]

    def frames(x):            # T_i(x) = R_i x + t_i, column vectors
        return torch.einsum("bnxy,bnhpy->bnhpx", rot, x) + trans[:, :, None, None, :]

    qg, kg, vg = frames(t["q_points"]), frames(t["k_points"]), frames(t["v_points"])
    gamma = 0.5 * _softplus(t["point_weight_raw"]) * math.sqrt(2.0 / (27.0 * P))     # [H]
    z = torch.einsum("birc,bjrc->bijc", t["z1"], t["z2"])                          # [B,N,N,Cz]
    bias = torch.einsum("bijc,ch->bhij", z, t["Wb"])                               # [B,H,N,N]
    scalar = torch.einsum("bihd,bjhd->bhij", q, k) / math.sqrt(3.0 * D)
    diff = qg[:, :, None] - kg[:, None, :]                                         # [B,i,j,H,P,3]
    sqdist = (diff * diff).sum(dim=(-1, -2)).permute(0, 3, 1, 2)                  # [B,H,i,j]
    logits = scalar + bias / math.sqrt(3.0) - gamma[None, :, None, None] * sqdist

    permitted = mask[:, :, None] & mask[:, None, :] & pair_mask                   # [B,i,j]
    perm = permitted[:, None].expand_as(logits)
    empty = ~permitted.any(dim=-1)                                                # [B,i]
    masked = torch.where(perm, logits, torch.full_like(logits, -math.inf))
    m = masked.amax(dim=-1, keepdim=True)
    m = torch.where(torch.isfinite(m), m, torch.zeros_like(m)).detach()
    safe = torch.where(perm, logits, torch.zeros_like(logits))
    e = torch.where(perm, torch.exp(safe - m), torch.zeros_like(logits))
    s = e.sum(dim=-1, keepdim=True)
    att = e / torch.where(s > 0, s, torch.ones_like(s))                          # [B,H,i,j]

    o_scalar = torch.einsum("bhij,bjhd->bihd", att, v)
    o_pair = torch.einsum("bhij,bijc->bihc", att, z)
    g_agg = torch.einsum("bhij,bjhqx->bihqx", att, vg)
    local = torch.einsum("biyx,bihqy->bihqx", rot, g_agg - trans[:, :, None, None, :])
    local = torch.where(empty[:, :, None, None, None], torch.zeros_like(local), local)
    lengths = torch.sqrt((local * local).sum(dim=-1) + eps)
    lengths = torch.where(empty[:, :, None, None], torch.zeros_like(lengths), lengths)
    features = torch.cat([
        o_scalar.reshape(B, N, -1),
        local[..., 0].reshape(B, N, -1),
        local[..., 1].reshape(B, N, -1),
        local[..., 2].reshape(B, N, -1),
        lengths.reshape(B, N, -1),
        o_pair.reshape(B, N, -1),
    ], dim=-1)
    update = features @ t["w_out"] + t["b_out"]
    update = torch.where(empty[:, :, None], torch.zeros_like(update), update)
    return update, local


def _tensors(inputs: dict, wrt: Iterable[str]):
    wrt = set(wrt)
    t = {key: torch.tensor(np.asarray(inputs[key], np.float64), dtype=torch.float64,
                           requires_grad=key in wrt) for key in FLOAT_KEYS}
    mask = torch.tensor(np.asarray(inputs["mask"]).astype(bool))
    B, N = mask.shape
    pm = inputs.get("pair_mask")
    pair_mask = (torch.ones((B, N, N), dtype=torch.bool) if pm is None
                 else torch.tensor(np.asarray(pm).astype(bool)))
    return t, mask, pair_mask


def forward(inputs: dict) -> Dict[str, np.ndarray]:
    """The restated forward (float64 NumPy outputs), for cross-checks."""
    t, mask, pair_mask = _tensors(inputs, ())
    with torch.no_grad():
        update, local = forward_torch(t, mask, pair_mask, float(inputs["eps"]))
    return {"update": update.numpy(), "local_points": local.numpy()}


def ipa_vjp(inputs: dict, d_update: np.ndarray, d_local: np.ndarray,
            wrt: Optional[Iterable[str]] = None) -> Dict[str, np.ndarray]:
    """Gradients of <d_update, update> + <d_local, local_points> with respect to
    the floating inputs `wrt` (default: all of FLOAT_KEYS), float64 NumPy."""
    wrt = tuple(FLOAT_KEYS if wrt is None else wrt)
    t, mask, pair_mask = _tensors(inputs, wrt)
    update, local = forward_torch(t, mask, pair_mask, float(inputs["eps"]))
    outs, cots = [], []
    for o, d in ((update, d_update), (local, d_local)):
        if o.requires_grad:              # (local points do not depend on w_out, b_out)
            outs.append(o)
            cots.append(torch.tensor(np.asarray(d, np.float64)))
    grads = torch.autograd.grad(outs, [t[key] for key in wrt], grad_outputs=cots, allow_unused=True)
    return {key: (g.numpy() if g is not None else np.zeros(t[key].shape))
            for key, g in zip(wrt, grads)}
