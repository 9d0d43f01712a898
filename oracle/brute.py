"""Pure-Python scalar brute force of each step, for tiny packs only.

TEST INFRASTRUCTURE ONLY. Written independently of ``mf_oracle`` (explicit
loops over samples, tokens, heads and channels, ``math`` scalars, no NumPy
vectorisation) so that an indexing or layout slip in the vectorised oracle shows
up as a mismatch. Same readings as the oracle; see ``oracle/__init__.py``.
"""

from __future__ import annotations

import math


def brute_pack(descs, rope_axes):
    """Enumerate tokens one by one: returns (cu_seqlens, pos_ids, tok_sample,
    tok_mod) as Python lists."""
    cu = [0]
    pos, ts, tm = [], [], []
    for s, d in enumerate(descs):
        F, Hg, Wg, L = tuple(d.as_tuple() if hasattr(d, "as_tuple") else d)[:4]
        count = 0
        for f in range(F):
            for h in range(Hg):
                for w in range(Wg):
                    pos.append((f, h, w))
                    ts.append(s)
                    tm.append(0)
                    count += 1
        first = Hg if Hg > Wg else Wg
        for j in range(L):
            p = first + j
            pos.append((p, p, p))
            ts.append(s)
            tm.append(1)
            count += 1
        cu.append(cu[-1] + count)
    return cu, pos, ts, tm


def brute_mod(c, W, hid):
    """mod[s][m][j][i] by explicit dot products."""
    S, C = len(c), len(c[0])
    out = [[[[0.0] * hid for _ in range(3)] for _ in range(2)] for _ in range(S)]
    for s in range(S):
        for m in range(2):
            for j in range(3):
                for i in range(hid):
                    col = (3 * m + j) * hid + i
                    acc = 0.0
                    for cc in range(C):
                        acc += float(c[s][cc]) * float(W[cc][col])
                    out[s][m][j][i] = acc
    return out


def brute_adaln_row(xrow, shift, scale, eps):
    n = len(xrow)
    mean = sum(float(v) for v in xrow) / n
    var = sum((float(v) - mean) ** 2 for v in xrow) / n
    inv = 1.0 / math.sqrt(var + eps)
    return [(float(xrow[i]) - mean) * inv * (1.0 + float(scale[i])) + float(shift[i])
            for i in range(n)]


def brute_rope_vec(vec, pos, rope_axes, base=10000.0):
    """Rotate one head vector channel by channel. Channel d belongs to axis
    chunk d // d_a; pair index inside the chunk is (d % d_a) // 2."""
    D = len(vec)
    d_a = 2 * (D // (2 * rope_axes))
    comps = (1, 2) if rope_axes == 2 else (0, 1, 2)
    out = [float(v) for v in vec]
    for d in range(0, D, 2):
        a = d // d_a
        if a >= rope_axes:
            continue  # leftover channels stay as they are
        i = (d % d_a) // 2
        ang = pos[comps[a]] * base ** (-(2.0 * i) / d_a)
        c, s = math.cos(ang), math.sin(ang)
        x0, x1 = float(vec[d]), float(vec[d + 1])
        out[d] = x0 * c - x1 * s
        out[d + 1] = x0 * s + x1 * c
    return out


def brute_attention(q, k, v, cu, scale=None):
    """Triple loop: for every sample, head and query row, the softmax over the
    sample's own keys. q, k, v are nested lists [T][H][D]."""
    T = len(q)
    H = len(q[0]) if T else 0
    D = len(q[0][0]) if T else 0
    if scale is None:
        scale = 1.0 / math.sqrt(D) if D else 1.0
    out = [[[0.0] * D for _ in range(H)] for _ in range(T)]
    for s in range(len(cu) - 1):
        lo, hi = cu[s], cu[s + 1]
        for h in range(H):
            for i in range(lo, hi):
                scores = []
                for j in range(lo, hi):
                    acc = 0.0
                    for d in range(D):
                        acc += float(q[i][h][d]) * float(k[j][h][d])
                    scores.append(acc * scale)
                mx = max(scores)
                e = [math.exp(sc - mx) for sc in scores]
                tot = sum(e)
                for d in range(D):
                    acc = 0.0
                    for jj, j in enumerate(range(lo, hi)):
                        acc += e[jj] * float(v[j][h][d])
                    out[i][h][d] = acc / tot
    return out


def brute_gate_row(xrow, orow, gate):
    return [float(xrow[i]) + float(gate[i]) * float(orow[i]) for i in range(len(xrow))]


def brute_linear_row(x_row, w_rows):
    """One output row of a linear map: one dot product per output feature."""
    return [sum(a * b for a, b in zip(x_row, w)) for w in w_rows]


def brute_gelu(v):
    return 0.5 * v * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (v + 0.044715 * v * v * v)))


def brute_mmdit_block(x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, descs, H, D, rope_axes,
                      base=10000.0, eps=1e-6):
    """The whole block, token by token and channel by channel, with no rounding
    of intermediates: adaLN, per-modality q/k/v, RoPE, per-sample attention,
    output projection and gate, second adaLN, GELU MLP and gate. Nested lists
    in, nested lists out ([T][H*D])."""
    cu, pos, ts, tm = brute_pack(descs, rope_axes)
    T = len(ts)
    hid = H * D

    def mod_vec(mod, t, j):
        return [float(mod[ts[t]][tm[t]][j][i]) for i in range(hid)]

    x1 = [brute_adaln_row(x[t], mod_vec(mod_attn, t, 0), mod_vec(mod_attn, t, 1), eps)
          for t in range(T)]
    q = [brute_linear_row(x1[t], Wq[tm[t]]) for t in range(T)]
    k = [brute_linear_row(x1[t], Wk[tm[t]]) for t in range(T)]
    v = [brute_linear_row(x1[t], Wv[tm[t]]) for t in range(T)]

    def heads(rows, rotate):
        out = []
        for t in range(T):
            hs = []
            for h in range(H):
                vec = rows[t][h * D:(h + 1) * D]
                hs.append(brute_rope_vec(vec, pos[t], rope_axes, base) if rotate else vec)
            out.append(hs)
        return out

    o = brute_attention(heads(q, True), heads(k, True), heads(v, False), cu)
    y = []
    for t in range(T):
        orow = [o[t][h][d] for h in range(H) for d in range(D)]
        a = brute_linear_row(orow, Wo[tm[t]])
        y1 = brute_gate_row(x[t], a, mod_vec(mod_attn, t, 2))
        x2 = brute_adaln_row(y1, mod_vec(mod_mlp, t, 0), mod_vec(mod_mlp, t, 1), eps)
        hmid = [brute_gelu(val) for val in brute_linear_row(x2, Wup[tm[t]])]
        m = brute_linear_row(hmid, Wdown[tm[t]])
        y.append(brute_gate_row(y1, m, mod_vec(mod_mlp, t, 2)))
    return y


def brute_attention_bwd(q, k, v, d_o, cu, scale=None):
    """dq, dk, dv of the per-sample attention by explicit loops: for each sample,
    head and query row, the softmax row p, then dp_j = <dO_i, v_j>,
    ds_j = p_j (dp_j - sum_l p_l dp_l), dq_i += scale ds_j k_j, dk_j += scale ds_j q_i,
    dv_j += p_j dO_i. Nested lists [T][H][D] in and out."""
    T = len(q)
    H = len(q[0]) if T else 0
    D = len(q[0][0]) if T else 0
    if scale is None:
        scale = 1.0 / math.sqrt(D) if D else 1.0
    dq = [[[0.0] * D for _ in range(H)] for _ in range(T)]
    dk = [[[0.0] * D for _ in range(H)] for _ in range(T)]
    dv = [[[0.0] * D for _ in range(H)] for _ in range(T)]
    for s in range(len(cu) - 1):
        lo, hi = cu[s], cu[s + 1]
        for h in range(H):
            for i in range(lo, hi):
                sc = [scale * sum(float(q[i][h][d]) * float(k[j][h][d]) for d in range(D))
                      for j in range(lo, hi)]
                mx = max(sc)
                e = [math.exp(a - mx) for a in sc]
                tot = sum(e)
                p = [a / tot for a in e]
                dp = [sum(float(d_o[i][h][d]) * float(v[j][h][d]) for d in range(D))
                      for j in range(lo, hi)]
                mean_dp = sum(pj * dpj for pj, dpj in zip(p, dp))
                for jj, j in enumerate(range(lo, hi)):
                    ds = p[jj] * (dp[jj] - mean_dp)
                    for d in range(D):
                        dq[i][h][d] += scale * ds * float(k[j][h][d])
                        dk[j][h][d] += scale * ds * float(q[i][h][d])
                        dv[j][h][d] += p[jj] * float(d_o[i][h][d])
    return dq, dk, dv
