"""Pure-Python scalar-loop restatement of the IPA aggregation core, for N <= 8.

Test infrastructure only (see the package docstring).  Written with nested
loops and the `math` module, sharing no helper with the vectorised oracle, so
that an index, sign or transpose slip in either one shows up as a mismatch.
Follows the BioTorch page "Invariant point attention (IPA)", section
"Required behavior", bullet by bullet.
"""
from __future__ import annotations

import math


def _softplus(x: float) -> float:
    # log(1 + e^x) without overflow
    if x > 0:
        return x + math.log1p(math.exp(-x))
    return math.log1p(math.exp(x))


def _frame(R, t, p):
    # column-vector convention: R @ p + t
    return [R[r][0] * p[0] + R[r][1] * p[1] + R[r][2] * p[2] + t[r] for r in range(3)]


def ipa_bruteforce(inp: dict) -> dict:
    """Loops over every (b, i, h, j).  `inp` holds nested lists or numpy arrays
    with the layout of `workloads.make_inputs`; pair values/bias are formed
    from the factors z1, z2 and the projection Wb."""
    q, k, v = inp["q"], inp["k"], inp["v"]
    qp, kp, vp = inp["q_points"], inp["k_points"], inp["v_points"]
    rot, tr = inp["rotation"], inp["translation"]
    z1, z2, Wb = inp["z1"], inp["z2"], inp["Wb"]
    raw, w_out, b_out = inp["point_weight_raw"], inp["w_out"], inp["b_out"]
    mask, pair_mask, eps = inp["mask"], inp["pair_mask"], float(inp["eps"])

    B, N, H, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Dv = len(v[0][0][0])
    P = len(qp[0][0][0])
    Q = len(vp[0][0][0])
    R = len(z1[0][0])
    Cz = len(z1[0][0][0])
    Cout = len(b_out)

    update = [[[0.0] * Cout for _ in range(N)] for _ in range(B)]
    local_out = [[[[[0.0] * 3 for _ in range(Q)] for _ in range(H)] for _ in range(N)] for _ in range(B)]
    attention = [[[[0.0] * N for _ in range(N)] for _ in range(H)] for _ in range(B)]

    for b in range(B):
        for i in range(N):
            permitted = []
            for j in range(N):
                pm = True if pair_mask is None else bool(pair_mask[b][i][j])
                permitted.append(bool(mask[b][i]) and bool(mask[b][j]) and pm)
            empty = not any(permitted)

            scal = [[0.0] * Dv for _ in range(H)]
            pair = [[0.0] * Cz for _ in range(H)]
            loc = [[[0.0] * 3 for _ in range(Q)] for _ in range(H)]
            for h in range(H):
                w = 0.5 * _softplus(float(raw[h])) * math.sqrt(2.0 / (27.0 * P))
                logit = [0.0] * N
                for j in range(N):
                    s = 0.0
                    for d in range(D):
                        s += q[b][i][h][d] * k[b][j][h][d]
                    s /= math.sqrt(3.0 * D)
                    bias = 0.0
                    for c in range(Cz):
                        zc = 0.0
                        for r in range(R):
                            zc += z1[b][i][r][c] * z2[b][j][r][c]
                        bias += zc * Wb[c][h]
                    s += bias / math.sqrt(3.0)
                    dist = 0.0
                    for p in range(P):
                        a = _frame(rot[b][i], tr[b][i], qp[b][i][h][p])
                        c3 = _frame(rot[b][j], tr[b][j], kp[b][j][h][p])
                        for x in range(3):
                            dist += (a[x] - c3[x]) ** 2
                    logit[j] = s - w * dist
                if empty:
                    continue
                mx = max(logit[j] for j in range(N) if permitted[j])
                ex = [math.exp(logit[j] - mx) if permitted[j] else 0.0 for j in range(N)]
                tot = sum(ex)
                att = [e / tot for e in ex]
                attention[b][h][i] = att
                for j in range(N):
                    if att[j] == 0.0:
                        continue
                    for d in range(Dv):
                        scal[h][d] += att[j] * v[b][j][h][d]
                    for c in range(Cz):
                        zc = 0.0
                        for r in range(R):
                            zc += z1[b][i][r][c] * z2[b][j][r][c]
                        pair[h][c] += att[j] * zc
                    for qq in range(Q):
                        g = _frame(rot[b][j], tr[b][j], vp[b][j][h][qq])
                        for x in range(3):
                            loc[h][qq][x] += att[j] * g[x]
                # back into the query frame: R_i^T (g - t_i)
                for qq in range(Q):
                    rel = [loc[h][qq][x] - tr[b][i][x] for x in range(3)]
                    loc[h][qq] = [sum(rot[b][i][y][x] * rel[y] for y in range(3)) for x in range(3)]
            if empty:
                continue
            feats = []
            for h in range(H):
                feats += scal[h]
            for x in range(3):
                for h in range(H):
                    for qq in range(Q):
                        feats.append(loc[h][qq][x])
            for h in range(H):
                for qq in range(Q):
                    feats.append(math.sqrt(sum(loc[h][qq][x] ** 2 for x in range(3)) + eps))
            for h in range(H):
                feats += pair[h]
            for o in range(Cout):
                acc = float(b_out[o])
                for f in range(len(feats)):
                    acc += feats[f] * w_out[f][o]
                update[b][i][o] = acc
            local_out[b][i] = loc
    return {"update": update, "local_points": local_out, "attention": attention}
