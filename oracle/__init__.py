"""CPU fp64 oracle of the IPA aggregation core -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import this package.  The product path (the CUDA library and
its Python binding) never imports, calls or links anything here, and this
package imports nothing from the product path.

What it computes is the IPA aggregation core as the BioTorch problem page
"Invariant point attention (IPA)" defines it (section "Required behavior"),
written out literally in float64 NumPy:

  * frames T_i(x) = rotation_i @ x + translation_i applied to every q/k/v
    point (column-vector convention);
  * logits L_ijh = q_ih.k_jh / sqrt(3D) + pair_bias_ijh / sqrt(3)
                   - 1/2 softplus(raw_h) sqrt(2/(27P)) sum_p |T_i q_p - T_j k_p|^2,
    squared distance without epsilon, negative sign;
  * key j permitted iff mask_i and mask_j and pair_mask_ij; stable softmax
    over j; an empty neighbourhood gives an all-zero attention row;
  * scalar, pair and global-point aggregation; inverse transform of the
    aggregated global value points into the query frame (rotation_i^T);
  * features [scalar | x | y | z | lengths | pair], each flattened
    head-major; lengths = sqrt(sum_xyz local^2 + eps), zero for an empty
    neighbourhood; update = features @ w_out + b_out, zero for an empty
    neighbourhood.

The pair representation of the FlashIPA form ("Flash Invariant Point
Attention": factors z1, z2 of shape (B, L, r, d), z_ij = z1_i^T z2_j) is
materialised densely per block of query rows by `ipa_forward_dense`, then
pair_bias_ijh = sum_c z_ij[c] Wb[c,h] (the per-head projection of the pair
representation; the pages leave its form open, this is the plain linear
reading, no bias term, since a per-head constant cancels in the softmax).
`ipa_forward_factorised` is an independent second arithmetic path through
the factors; the two must agree to rounding.

Pins (see tests/test_oracle.py): closed form of the page's worked example
"Nearby frames receive more weight"; invariance under a global rigid motion
(page: "All three outputs are invariant ..."); attention row sums in
{0, 1}; exact structural zeros; the scalar-only and distance-only special
cases against torch's scaled_dot_product_attention and scipy's cdist +
softmax; the identity-neighbourhood closed form; a pure-Python brute force
for N <= 8; dense == factorised.  The pages print no expected output values,
so absolute end-to-end numbers are pinned only through these checks.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "softplus", "point_weight", "apply_frames", "invariant_point_attention",
    "ipa_forward_dense", "ipa_forward_factorised", "feature_width",
]


# --------------------------------------------------------------------------
# elementary pieces ("Required behavior", logit and softplus bullets)
# --------------------------------------------------------------------------
def softplus(x):
    """softplus(x) = log(1 + exp(x)) written without overflow:
    max(x, 0) + log1p(exp(-|x|))."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def point_weight(point_weight_raw, P: int):
    """Per-head distance weight 1/2 * softplus(raw_h) * sqrt(2 / (27 P)).

    P is the number of query/key points (value points do not enter the logit)."""
    return 0.5 * softplus(point_weight_raw) * math.sqrt(2.0 / (27.0 * P))


def apply_frames(rotation, translation, points):
    """T_i(x) = rotation_i @ x + translation_i for points [..., N, H, P, 3].

    rotation [..., N, 3, 3], translation [..., N, 3]; column-vector convention."""
    return (np.einsum("...nxy,...nhpy->...nhpx", rotation, points)
            + translation[..., :, None, None, :])


def feature_width(H, Dv, Q, Cz):
    """F = H * (Dv + 4 Q + Cz)."""
    return H * (Dv + 4 * Q + Cz)


# --------------------------------------------------------------------------
# one batch element, a block of query rows, dense pair tensors
# --------------------------------------------------------------------------
def _core_rows(q, k, v, qg, kg, vg, rot, trans, mask, pair_mask_rows, rows,
               pair_bias_rows, pair_values_rows, gamma, w_out, b_out, eps,
               want_attention):
    """Outputs for query rows `rows` of one batch element.

    q [N,H,D], k [N,H,D], v [N,H,Dv]; qg/kg [N,H,P,3] and vg [N,H,Q,3] are
    global points; pair_bias_rows [n,N,H]; pair_values_rows [n,N,Cz];
    pair_mask_rows [n,N] bool.  Returns a dict of per-row outputs."""
    N, H, D = q.shape
    rows = np.asarray(rows)
    n = len(rows)

    # logit terms, [n, H, N]
    scalar = np.einsum("ihd,jhd->ihj", q[rows], k) / math.sqrt(3.0 * D)
    bias = np.transpose(pair_bias_rows, (0, 2, 1)) / math.sqrt(3.0)
    diff = qg[rows][:, None, :, :, :] - kg[None, :, :, :, :]     # [n, N, H, P, 3]
    sqdist = np.sum(diff * diff, axis=(3, 4))                    # [n, N, H]
    sqdist = np.transpose(sqdist, (0, 2, 1))                     # [n, H, N]
    logits = scalar + bias - gamma[None, :, None] * sqdist

    # masks: permit j iff mask_i and mask_j and pair_mask_ij
    permitted = mask[rows][:, None] & mask[None, :] & pair_mask_rows      # [n, N]
    perm = np.broadcast_to(permitted[:, None, :], logits.shape)
    empty = ~permitted.any(axis=1)                                         # [n]

    # stable softmax over permitted j; all-zero row for an empty neighbourhood
    masked = np.where(perm, logits, -np.inf)
    m = masked.max(axis=2, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.where(perm, np.exp(masked - m_safe), 0.0)
    s = e.sum(axis=2, keepdims=True)
    att = np.where(s > 0, e / np.where(s > 0, s, 1.0), 0.0)               # [n, H, N]
    with np.errstate(divide="ignore"):
        lse = np.where(s[..., 0] > 0, m_safe[..., 0] + np.log(np.where(s[..., 0] > 0, s[..., 0], 1.0)), -np.inf)

    # aggregation
    o_scalar = np.einsum("ihj,jhd->ihd", att, v)                          # [n, H, Dv]
    o_pair = np.einsum("ihj,ijc->ihc", att, pair_values_rows)             # [n, H, Cz]
    g_agg = np.einsum("ihj,jhqx->ihqx", att, vg)                          # [n, H, Q, 3]
    local = np.einsum("iyx,ihqy->ihqx", rot[rows], g_agg - trans[rows][:, None, None, :])
    local = np.where(empty[:, None, None, None], 0.0, local)
    lengths = np.sqrt(np.sum(local * local, axis=-1) + eps)
    lengths = np.where(empty[:, None, None], 0.0, lengths)

    # features, head-major flatten of each block, in the page's order
    features = np.concatenate([
        o_scalar.reshape(n, -1),
        local[..., 0].reshape(n, -1),
        local[..., 1].reshape(n, -1),
        local[..., 2].reshape(n, -1),
        lengths.reshape(n, -1),
        o_pair.reshape(n, -1),
    ], axis=1)
    update = features @ w_out + b_out
    update = np.where(empty[:, None], 0.0, update)

    out = {"update": update, "local_points": local, "lse": lse, "empty": empty,
           "features": features}
    if want_attention:
        out["attention"] = att
    return out


def _global_points(inputs):
    rot = np.asarray(inputs["rotation"], np.float64)
    trans = np.asarray(inputs["translation"], np.float64)
    qg = apply_frames(rot, trans, np.asarray(inputs["q_points"], np.float64))
    kg = apply_frames(rot, trans, np.asarray(inputs["k_points"], np.float64))
    vg = apply_frames(rot, trans, np.asarray(inputs["v_points"], np.float64))
    return rot, trans, qg, kg, vg


def _pair_mask_rows(pair_mask, b, rows, N):
    if pair_mask is None:
        return np.ones((len(rows), N), dtype=bool)
    return np.asarray(pair_mask[b])[np.asarray(rows)].astype(bool)


def _alloc_outputs(B, N, H, Q, Cout, nrows, want_attention):
    out = {
        "update": np.zeros((B, nrows, Cout)),
        "local_points": np.zeros((B, nrows, H, Q, 3)),
        "lse": np.full((B, H, nrows), -np.inf),
    }
    if want_attention:
        out["attention"] = np.zeros((B, H, nrows, N))
    return out


def _store(out, b, sl, res, want_attention):
    out["update"][b, sl] = res["update"]
    out["local_points"][b, sl] = res["local_points"]
    out["lse"][b, :, sl] = np.transpose(res["lse"], (1, 0))
    if want_attention:
        out["attention"][b, :, sl, :] = np.transpose(res["attention"], (1, 0, 2))


def _block_rows(N, H, P, Cz):
    # keep the [n, N, H, P, 3] difference tensor and the [n, N, Cz] pair block
    # around 128 MB each
    per_row = max(N * H * P * 3, N * Cz, N * H) * 8
    return int(max(1, min(256, (128 << 20) // per_row)))


# --------------------------------------------------------------------------
# the page's own signature, dense pair inputs
# --------------------------------------------------------------------------
def invariant_point_attention(activations: dict, parameters: dict, masks: dict,
                              structure: dict, eps: float = 1e-8) -> dict:
    """The page's function signature with dense pair inputs.

    activations: q [B,N,H,D], k [B,N,H,D], v [B,N,H,Dv],
                 q_points [B,N,H,P,3], k_points [B,N,H,P,3], v_points [B,N,H,Q,3],
                 pair_bias [B,N,N,H], pair_values [B,N,N,Cz]
    parameters:  point_weight_raw [H], w_out [F,Cout], b_out [Cout]
    masks:       mask [B,N] (True = valid), pair_mask [B,N,N] or None
    structure:   rotation [B,N,3,3], translation [B,N,3]
    Returns update [B,N,Cout], attention [B,H,N,N], local_points [B,N,H,Q,3]
    (and lse [B,H,N], the natural-log logsumexp of the permitted logits)."""
    inputs = dict(activations)
    inputs.update(parameters)
    inputs.update(structure)
    inputs["mask"] = masks["mask"]
    inputs["pair_mask"] = masks.get("pair_mask")
    q = np.asarray(inputs["q"], np.float64)
    B, N, H, _ = q.shape
    Q = np.asarray(inputs["v_points"]).shape[3]
    P = np.asarray(inputs["q_points"]).shape[3]
    w_out = np.asarray(inputs["w_out"], np.float64)
    b_out = np.asarray(inputs["b_out"], np.float64)
    gamma = point_weight(np.asarray(inputs["point_weight_raw"], np.float64), P)
    rot, trans, qg, kg, vg = _global_points(inputs)
    mask = np.asarray(inputs["mask"]).astype(bool)
    out = _alloc_outputs(B, N, H, Q, w_out.shape[1], N, True)
    for b in range(B):
        rows = np.arange(N)
        res = _core_rows(q[b], np.asarray(inputs["k"], np.float64)[b],
                         np.asarray(inputs["v"], np.float64)[b],
                         qg[b], kg[b], vg[b], rot[b], trans[b], mask[b],
                         _pair_mask_rows(inputs["pair_mask"], b, rows, N), rows,
                         np.asarray(inputs["pair_bias"], np.float64)[b],
                         np.asarray(inputs["pair_values"], np.float64)[b],
                         gamma, w_out, b_out, eps, True)
        _store(out, b, slice(0, N), res, True)
    return out


# --------------------------------------------------------------------------
# FlashIPA inputs (factors z1, z2 and projection Wb), dense materialisation
# --------------------------------------------------------------------------
def ipa_forward_dense(inputs: dict, rows: Optional[Sequence[int]] = None,
                      want_attention: bool = False) -> dict:
    """IPA core on factorised pair inputs, materialising the dense pair tensor.

    For every block of query rows it builds z_ij[c] = sum_r z1[i,r,c] z2[j,r,c]
    and pair_bias_ijh = sum_c z_ij[c] Wb[c,h] explicitly, then follows the page's
    definition.  `rows` (same for every batch element) restricts the outputs to
    those query rows; every output row depends on all keys, so a subset is
    exact on its own.  Input layout as `workloads.make_inputs` documents."""
    q = np.asarray(inputs["q"], np.float64)
    k = np.asarray(inputs["k"], np.float64)
    v = np.asarray(inputs["v"], np.float64)
    z1 = np.asarray(inputs["z1"], np.float64)
    z2 = np.asarray(inputs["z2"], np.float64)
    Wb = np.asarray(inputs["Wb"], np.float64)
    w_out = np.asarray(inputs["w_out"], np.float64)
    b_out = np.asarray(inputs["b_out"], np.float64)
    B, N, H, _ = q.shape
    P = np.asarray(inputs["q_points"]).shape[3]
    Q = np.asarray(inputs["v_points"]).shape[3]
    Cz = z1.shape[3]
    gamma = point_weight(np.asarray(inputs["point_weight_raw"], np.float64), P)
    rot, trans, qg, kg, vg = _global_points(inputs)
    mask = np.asarray(inputs["mask"]).astype(bool)
    eps = float(inputs["eps"])
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = _alloc_outputs(B, N, H, Q, w_out.shape[1], len(rows), want_attention)
    blk = _block_rows(N, H, P, Cz)
    for b in range(B):
        for s in range(0, len(rows), blk):
            r = rows[s:s + blk]
            pair_values = np.einsum("irc,jrc->ijc", z1[b, r], z2[b])     # [n, N, Cz]
            pair_bias = pair_values @ Wb                                  # [n, N, H]
            res = _core_rows(q[b], k[b], v[b], qg[b], kg[b], vg[b], rot[b], trans[b],
                             mask[b], _pair_mask_rows(inputs["pair_mask"], b, r, N), r,
                             pair_bias, pair_values, gamma, w_out, b_out, eps,
                             want_attention)
            _store(out, b, slice(s, s + len(r)), res, want_attention)
    return out


# --------------------------------------------------------------------------
# second, factorised arithmetic path (no N x N x Cz tensor)
# --------------------------------------------------------------------------
def ipa_forward_factorised(inputs: dict, rows: Optional[Sequence[int]] = None,
                           want_attention: bool = False) -> dict:
    """Same outputs as `ipa_forward_dense`, computed through the factors.

    pair bias:  sum_c z_ij[c] Wb[c,h] = sum_{r,c} (z1[i,r,c] Wb[c,h]) z2[j,r,c]
    pair value: sum_j a_ij z_ij[c]  = sum_r z1[i,r,c] (sum_j a_ij z2[j,r,c])
    The squared distance is taken directly (no norm expansion)."""
    q = np.asarray(inputs["q"], np.float64)
    k = np.asarray(inputs["k"], np.float64)
    v = np.asarray(inputs["v"], np.float64)
    z1 = np.asarray(inputs["z1"], np.float64)
    z2 = np.asarray(inputs["z2"], np.float64)
    Wb = np.asarray(inputs["Wb"], np.float64)
    w_out = np.asarray(inputs["w_out"], np.float64)
    b_out = np.asarray(inputs["b_out"], np.float64)
    B, N, H, D = q.shape
    P = np.asarray(inputs["q_points"]).shape[3]
    Q = np.asarray(inputs["v_points"]).shape[3]
    Cz = z1.shape[3]
    gamma = point_weight(np.asarray(inputs["point_weight_raw"], np.float64), P)
    rot, trans, qg, kg, vg = _global_points(inputs)
    mask = np.asarray(inputs["mask"]).astype(bool)
    eps = float(inputs["eps"])
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = _alloc_outputs(B, N, H, Q, w_out.shape[1], len(rows), want_attention)
    blk = _block_rows(N, H, P, Cz)
    for b in range(B):
        for s in range(0, len(rows), blk):
            r = rows[s:s + blk]
            n = len(r)
            u = np.einsum("irc,ch->ihrc", z1[b, r], Wb)                   # z1 (.) Wb
            bias = np.einsum("ihrc,jrc->ihj", u, z2[b]) / math.sqrt(3.0)  # [n, H, N]
            scalar = np.einsum("ihd,jhd->ihj", q[b, r], k[b]) / math.sqrt(3.0 * D)
            sq = np.zeros((n, H, N))
            for p in range(P):
                for x in range(3):
                    dlt = qg[b, r, :, p, x][:, :, None] - kg[b, :, :, p, x].T[None, :, :]
                    sq += dlt * dlt
            logits = scalar + bias - gamma[None, :, None] * sq
            pm = _pair_mask_rows(inputs["pair_mask"], b, r, N)
            permitted = mask[b, r][:, None] & mask[b][None, :] & pm
            empty = ~permitted.any(axis=1)
            perm = np.broadcast_to(permitted[:, None, :], logits.shape)
            m = np.where(perm, logits, -np.inf).max(axis=2, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            e = np.where(perm, np.exp(np.where(perm, logits, 0.0) - m), 0.0)
            ssum = e.sum(axis=2, keepdims=True)
            att = e / np.where(ssum > 0, ssum, 1.0)
            with np.errstate(divide="ignore"):
                lse = np.where(ssum[..., 0] > 0, m[..., 0] + np.log(np.where(ssum[..., 0] > 0, ssum[..., 0], 1.0)), -np.inf)
            o_scalar = np.einsum("ihj,jhd->ihd", att, v[b])
            az2 = np.einsum("ihj,jrc->ihrc", att, z2[b])
            o_pair = np.einsum("irc,ihrc->ihc", z1[b, r], az2)
            g_agg = np.einsum("ihj,jhqx->ihqx", att, vg[b])
            rel = g_agg - trans[b, r][:, None, None, :]
            local = np.einsum("iyx,ihqy->ihqx", rot[b, r], rel)
            local[empty] = 0.0
            lengths = np.sqrt((local ** 2).sum(-1) + eps)
            lengths[empty] = 0.0
            feats = np.concatenate([o_scalar.reshape(n, -1), local[..., 0].reshape(n, -1),
                                    local[..., 1].reshape(n, -1), local[..., 2].reshape(n, -1),
                                    lengths.reshape(n, -1), o_pair.reshape(n, -1)], axis=1)
            upd = feats @ w_out + b_out
            upd[empty] = 0.0
            sl = slice(s, s + n)
            out["update"][b, sl] = upd
            out["local_points"][b, sl] = local
            out["lse"][b, :, sl] = lse.T
            if want_attention:
                out["attention"][b, :, sl, :] = np.transpose(att, (1, 0, 2))
    return out
