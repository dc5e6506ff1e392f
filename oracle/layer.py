"""The IPA layer around the aggregation core -- TEST INFRASTRUCTURE ONLY.

Same import rules as the `oracle` package: only `tests/`,
`__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` may use it;
it imports nothing from the product path.

The BioTorch page "Invariant point attention (IPA)" (Required behavior)
defines the core as starting after the input projections and ending before
any residual or frame update, and asks not to invent weights for them.  This
module is the plainest layer around that core, every weight supplied by the
caller (nothing is learned or invented here):

  1. one affine projection of the single representation s [B,N,Cs]:
     X = s @ W_in + b_in, split in this order into q [H,D], k [H,D], v [H,Dv],
     q_points [H,P,3], k_points [H,P,3], v_points [H,Q,3] (LOCAL points, the
     bias being the learned point-projection bias the page mentions), and the
     FlashIPA pair factors z1 [R,Cz], z2 [R,Cz] ("Flash Invariant Point
     Attention": factors of shape (B, L, r, d) from the 1D representation);
     each block is a row-major reshape of its columns;
  2. the core (oracle.ipa_forward_dense) with Wb, point_weight_raw, the masks,
     w_out [F,Cs], b_out [Cs];
  3. the residual s' = s + update;
  4. a frame update from s': [b, c, d, tx, ty, tz] = s' @ W_bb + b_bb, the
     rotation of the unit quaternion (1, b, c, d) / |(1, b, c, d)| and the
     translation (tx, ty, tz) in the residue's own frame, composed on the
     right: R' = R dR, t' = R dt + t; a masked residue keeps its frame.

Pinned in tests/test_oracle_layer.py: with W_in selecting given core inputs
the layer reduces to the core; zero frame update keeps the frames; a constant
update composes as scipy's rotations do; s' is invariant and the new frames
move with a global rigid motion.
"""
from __future__ import annotations

import numpy as np

import oracle

__all__ = ["layer_widths", "quaternion_rotation", "ipa_layer"]


def layer_widths(H, D, Dv, P, Q, Cz, R):
    """Column blocks of X = s @ W_in + b_in, in order: name -> (start, width)."""
    blocks = [("q", H * D), ("k", H * D), ("v", H * Dv), ("q_points", H * P * 3),
              ("k_points", H * P * 3), ("v_points", H * Q * 3), ("z1", R * Cz), ("z2", R * Cz)]
    out, o = {}, 0
    for name, w in blocks:
        out[name] = (o, w)
        o += w
    return out, o


def quaternion_rotation(b, c, d):
    """Rotation matrix of the unit quaternion (1, b, c, d) / |(1, b, c, d)|
    (scalar first), column-vector convention."""
    b, c, d = (np.asarray(x, np.float64) for x in (b, c, d))
    n = np.sqrt(1.0 + b * b + c * c + d * d)
    w, x, y, z = 1.0 / n, b / n, c / n, d / n
    R = np.empty(b.shape + (3, 3))
    R[..., 0, 0] = w * w + x * x - y * y - z * z
    R[..., 0, 1] = 2 * (x * y - w * z)
    R[..., 0, 2] = 2 * (x * z + w * y)
    R[..., 1, 0] = 2 * (x * y + w * z)
    R[..., 1, 1] = w * w - x * x + y * y - z * z
    R[..., 1, 2] = 2 * (y * z - w * x)
    R[..., 2, 0] = 2 * (x * z - w * y)
    R[..., 2, 1] = 2 * (y * z + w * x)
    R[..., 2, 2] = w * w - x * x - y * y + z * z
    return R


def ipa_layer(inp: dict, dims: dict) -> dict:
    """inp: s [B,N,Cs], W_in [Cs,Din], b_in [Din], rotation [B,N,3,3],
    translation [B,N,3], mask [B,N], pair_mask or None, Wb [Cz,H],
    point_weight_raw [H], w_out [F,Cs], b_out [Cs], W_bb [Cs,6], b_bb [6], eps.
    dims: H, D, Dv, P, Q, Cz, R.  Returns s_new [B,N,Cs], rotation, translation,
    local_points and the core inputs it formed."""
    s = np.asarray(inp["s"], np.float64)
    B, N, Cs = s.shape
    H, D, Dv, P, Q, Cz, R = (dims[k] for k in ("H", "D", "Dv", "P", "Q", "Cz", "R"))
    blocks, Din = layer_widths(H, D, Dv, P, Q, Cz, R)
    X = s @ np.asarray(inp["W_in"], np.float64) + np.asarray(inp["b_in"], np.float64)
    assert X.shape[-1] == Din
    shapes = {"q": (H, D), "k": (H, D), "v": (H, Dv), "q_points": (H, P, 3), "k_points": (H, P, 3),
              "v_points": (H, Q, 3), "z1": (R, Cz), "z2": (R, Cz)}
    core_in = {name: X[..., o:o + w].reshape((B, N) + shapes[name]) for name, (o, w) in blocks.items()}
    for key in ("rotation", "translation", "mask", "pair_mask", "Wb", "point_weight_raw", "w_out", "b_out", "eps"):
        core_in[key] = inp.get(key)
    out = oracle.ipa_forward_dense(core_in)
    s_new = s + out["update"]
    u = s_new @ np.asarray(inp["W_bb"], np.float64) + np.asarray(inp["b_bb"], np.float64)
    dR = quaternion_rotation(u[..., 0], u[..., 1], u[..., 2])
    rot = np.asarray(inp["rotation"], np.float64)
    trans = np.asarray(inp["translation"], np.float64)
    rot_new = np.einsum("bnxy,bnyz->bnxz", rot, dR)
    trans_new = np.einsum("bnxy,bny->bnx", rot, u[..., 3:6]) + trans
    keep = ~np.asarray(inp["mask"]).astype(bool)
    rot_new[keep] = rot[keep]
    trans_new[keep] = trans[keep]
    return {"s": s_new, "rotation": rot_new, "translation": trans_new,
            "local_points": out["local_points"], "core_inputs": core_in}
