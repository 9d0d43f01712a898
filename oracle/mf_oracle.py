"""Plain fp64 NumPy definition of each step of the packed joint-attention block.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): slow, obviously correct,
no blocking or fusion beyond what each definition states. Inputs arrive as
float32 arrays holding exact bf16 values; every computation is float64.
"""

from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

MOD_IMG = 0  # modality id of image-latent tokens
MOD_TXT = 1  # modality id of text tokens

SHIFT, SCALE, GATE = 0, 1, 2  # order of the three modulation vectors


# ---------------------------------------------------------------------------
# Pack metadata  ([pack], [rope], [edit])
# ---------------------------------------------------------------------------
def pack_build(descs: Sequence, rope_axes: int):
    """Per-sample cumulative offsets and per-token ids of a native-resolution pack.

    [pack]: samples share one flat token buffer; sample s owns tokens
    ``cu_seqlens[s] .. cu_seqlens[s+1]-1``.

    Readings (the pages give no layout):
      * inside a sample, image tokens come first, frame-major then row-major
        (f, h, w), followed by the text tokens;
      * an image token's position is (f, h, w); for 2D packs f = 0 ([rope]),
        for edit packs the frame index tells source (0) from target (1) ([edit]);
      * text token j sits on a 1D axis after the image grid: p = max(Hg, Wg) + j
        on every axis, i.e. position (p, p, p);
      * a text-only segment (frames = 0, empty grid) has positions 0, 1, 2, ...

    Returns a dict with int32 ``cu_seqlens`` [S+1], int32 ``pos_ids`` [T][3]
    (f, h, w), int32 ``tok_sample`` [T], uint8 ``tok_mod`` [T] (0 image,
    1 text) and ``T``.
    """
    descs = [tuple(d.as_tuple()) if hasattr(d, "as_tuple") else tuple(d) for d in descs]
    if rope_axes not in (2, 3):
        raise ValueError("rope_axes must be 2 or 3")
    n = []
    for (F, Hg, Wg, L, *_rest) in descs:
        if min(F, Hg, Wg, L) < 0:
            raise ValueError("negative descriptor field")
        if rope_axes == 2 and F > 1:
            raise ValueError("a 2D pack holds one frame per sample")
        if rope_axes == 3 and F > 2:
            raise ValueError("an edit pack holds at most two frames per sample")
        n.append(F * Hg * Wg + L)
    S = len(descs)
    cu = np.zeros(S + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(n, dtype=np.int64))
    T = int(cu[-1])
    pos = np.zeros((T, 3), dtype=np.int32)
    tok_sample = np.zeros(T, dtype=np.int32)
    tok_mod = np.zeros(T, dtype=np.uint8)
    for s, (F, Hg, Wg, L, *_rest) in enumerate(descs):
        start = int(cu[s])
        n_img = F * Hg * Wg
        f, h, w = np.meshgrid(np.arange(F), np.arange(Hg), np.arange(Wg), indexing="ij")
        pos[start:start + n_img, 0] = f.ravel()
        pos[start:start + n_img, 1] = h.ravel()
        pos[start:start + n_img, 2] = w.ravel()
        p = max(Hg, Wg) + np.arange(L)
        pos[start + n_img:start + n_img + L, :] = p[:, None]
        tok_sample[start:start + n_img + L] = s
        tok_mod[start + n_img:start + n_img + L] = MOD_TXT
    return dict(cu_seqlens=cu.astype(np.int32), pos_ids=pos, tok_sample=tok_sample,
                tok_mod=tok_mod, T=T)


# ---------------------------------------------------------------------------
# Modality-specific adaptive LayerNorm  ([norm], [fuse])
# ---------------------------------------------------------------------------
def adaln_params(c: np.ndarray, W: np.ndarray, hid: int) -> np.ndarray:
    """Per-sample, per-modality shift / scale / gate vectors.

    Reading: a plain linear map of the conditioning vector (no bias, no
    activation): ``mod[s][m][j][i] = sum_c c[s][c] * W[c][(3*m + j)*hid + i]``
    with m in {image, text} and j in {shift, scale, gate}.
    Returns float64 [S][2][3][hid].
    """
    c = np.asarray(c, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    S = c.shape[0]
    if W.shape != (c.shape[1], 6 * hid):
        raise ValueError("W must be [C][6*hid]")
    return (c @ W).reshape(S, 2, 3, hid)


def layer_norm_rows(x: np.ndarray, eps: float) -> np.ndarray:
    """LayerNorm without affine parameters over the last axis: population
    variance, ``(x - mean) / sqrt(var + eps)``."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = np.mean((x - mu) ** 2, axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def adaln_modulate(x, mod, tok_sample, tok_mod, eps: float = 1e-6, rows=None):
    """``x_mod[t] = LN(x[t]) * (1 + scale[s, m]) + shift[s, m]`` with s the
    token's sample and m its modality ([norm]). Reading: eps = 1e-6, no affine
    LayerNorm parameters. ``rows`` restricts the output to those token rows."""
    x = np.asarray(x, dtype=np.float64)
    tok_sample = np.asarray(tok_sample)
    tok_mod = np.asarray(tok_mod)
    if rows is not None:
        x, tok_sample, tok_mod = x[rows], tok_sample[rows], tok_mod[rows]
    ln = layer_norm_rows(x, eps)
    shift = mod[tok_sample, tok_mod, SHIFT]
    scale = mod[tok_sample, tok_mod, SCALE]
    return ln * (1.0 + scale) + shift


# ---------------------------------------------------------------------------
# Per-sample 2D / 3D rotary embedding  ([rope], [edit])
# ---------------------------------------------------------------------------
def rope_split(D: int, rope_axes: int) -> int:
    """Channels given to each axis. Reading: head_dim is split evenly across
    the axes in whole pairs, ``d_a = 2 * floor(D / (2 * axes))``; the chunks are
    contiguous in axis order ((h, w) for 2D, (f, h, w) for 3D) and any leftover
    channels at the end are not rotated (D = 128, 3D: 42 | 42 | 42 | 2 kept)."""
    if D % 2:
        raise ValueError("head_dim must be even")
    return 2 * (D // (2 * rope_axes))


def rope_pair_angles(pos_ids: np.ndarray, D: int, rope_axes: int, base: float = 10000.0):
    """Rotation angle of every channel pair for every token: float64 [T][D/2].

    Pair i of an axis chunk of width d_a turns by
    ``theta = pos_axis * base ** (-2 i / d_a)`` (reading: base 10000); pairs past
    the last chunk get angle 0."""
    pos_ids = np.asarray(pos_ids)
    d_a = rope_split(D, rope_axes)
    comps = (1, 2) if rope_axes == 2 else (0, 1, 2)  # which (f, h, w) entry drives each chunk
    inv_freq = np.power(float(base), -np.arange(0, d_a, 2, dtype=np.float64) / d_a)  # [d_a/2]
    theta = np.zeros((pos_ids.shape[0], D // 2), dtype=np.float64)
    for a, comp in enumerate(comps):
        p = pos_ids[:, comp].astype(np.float64)
        theta[:, a * (d_a // 2):(a + 1) * (d_a // 2)] = p[:, None] * inv_freq[None, :]
    return theta


def rope_apply(x, pos_ids, rope_axes: int, base: float = 10000.0, rows=None):
    """Rotate interleaved channel pairs ``(x[2i], x[2i+1])`` of every head by the
    token's angles: ``x0' = x0 cos - x1 sin``, ``x1' = x0 sin + x1 cos``.
    Reading: pairs are adjacent channels. x is [T][H][D]; returns float64."""
    x = np.asarray(x, dtype=np.float64)
    pos_ids = np.asarray(pos_ids)
    if rows is not None:
        x, pos_ids = x[rows], pos_ids[rows]
    D = x.shape[-1]
    theta = rope_pair_angles(pos_ids, D, rope_axes, base)[:, None, :]  # [T][1][D/2]
    cos, sin = np.cos(theta), np.sin(theta)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * cos - x1 * sin
    out[..., 1::2] = x0 * sin + x1 * cos
    return out


# ---------------------------------------------------------------------------
# Block-diagonal variable-length attention  ([pack], [norm])
# ---------------------------------------------------------------------------
def varlen_attention(q, k, v, cu_seqlens, scale: Optional[float] = None,
                     rows=None, chunk: int = 2048):
    """Joint self-attention inside each sample of the pack: for sample s and
    head h, ``O = softmax(Q K^T * scale) V`` over the sample's own tokens (image
    and text together, no mask inside a sample, nothing across samples).
    Reading: scale = 1/sqrt(D).

    q, k, v: [T][H][D]. Returns (O float64 [T][H][D], lse float64 [H][T]) where
    ``lse = log sum_j exp(s_ij)`` (natural log). With ``rows`` (sorted token
    indices) only those query rows are computed; O is then [len(rows)][H][D] and
    lse [H][len(rows)]. Query rows are processed ``chunk`` at a time only to
    bound memory."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((rows.shape[0], H, D), dtype=np.float64)
    lse = np.zeros((H, rows.shape[0]), dtype=np.float64)
    sample_of_row = np.searchsorted(cu, rows, side="right") - 1
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        sel = np.nonzero(sample_of_row == s)[0]
        if sel.size == 0 or hi == lo:
            continue
        for h in range(H):
            Ks = k[lo:hi, h, :]
            Vs = v[lo:hi, h, :]
            for c0 in range(0, sel.size, chunk):
                idx = sel[c0:c0 + chunk]
                Qc = q[rows[idx], h, :]
                Sc = (Qc @ Ks.T) * scale
                m = Sc.max(axis=1, keepdims=True)
                P = np.exp(Sc - m)
                l = P.sum(axis=1, keepdims=True)
                out[idx, h, :] = (P @ Vs) / l
                lse[h, idx] = (m + np.log(l))[:, 0]
    return out, lse


# ---------------------------------------------------------------------------
# Gated residual  ([fuse])
# ---------------------------------------------------------------------------
def varlen_attention_bwd(q, k, v, d_o, cu_seqlens, scale: Optional[float] = None):
    """Gradients of the packed joint attention with respect to q, k and v.

    For sample s and head h, with S = scale Q K^T, P = softmax(S) (rows),
    O = P V and the output gradient dO (chain rule, written out):
        dV = P^T dO
        dP = dO V^T
        dS = P * (dP - rowsum(dO * O))      (the softmax Jacobian, row by row)
        dQ = scale dS K,  dK = scale dS^T Q
    Nothing flows across samples (block-diagonal, like the forward). q, k, v,
    d_o: [T][H][D]. Returns float64 (dq, dk, dv), each [T][H][D].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d_o = np.asarray(d_o, dtype=np.float64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        if hi == lo:
            continue
        for h in range(H):
            Q, K, V, dO = q[lo:hi, h], k[lo:hi, h], v[lo:hi, h], d_o[lo:hi, h]
            S = (Q @ K.T) * scale
            P = np.exp(S - S.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            O = P @ V
            dv[lo:hi, h] = P.T @ dO
            dP = dO @ V.T
            dS = P * (dP - (dO * O).sum(axis=1, keepdims=True))
            dq[lo:hi, h] = scale * (dS @ K)
            dk[lo:hi, h] = scale * (dS.T @ Q)
    return dq, dk, dv


def gated_residual(x, o, mod, tok_sample, tok_mod, rows=None):
    """``y[t] = x[t] + gate[s, m] * O[t]`` with O viewed as [T][H*D] (head-major
    columns). Reading: the gate multiplies the attention branch and is added to
    the block input (adaLN-zero form; no output projection on this path)."""
    x = np.asarray(x, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64).reshape(x.shape[0], -1)
    tok_sample = np.asarray(tok_sample)
    tok_mod = np.asarray(tok_mod)
    if rows is not None:
        x, o, tok_sample, tok_mod = x[rows], o[rows], tok_sample[rows], tok_mod[rows]
    gate = mod[tok_sample, tok_mod, GATE]
    return x + gate * o


# ---------------------------------------------------------------------------
# The whole block
# ---------------------------------------------------------------------------
def block_fwd(x, q, k, v, mod, pack, rope_axes: int, base: float = 10000.0,
              eps: float = 1e-6, rows=None):
    """adaLN modulation, RoPE on Q and K, joint varlen attention and the gated
    residual, in the order the fused chain names them ([fuse]). Returns
    (x_mod, y, O) in float64, restricted to ``rows`` when given."""
    tok_sample, tok_mod = pack["tok_sample"], pack["tok_mod"]
    x_mod = adaln_modulate(x, mod, tok_sample, tok_mod, eps, rows=rows)
    q_r = rope_apply(q, pack["pos_ids"], rope_axes, base, rows=rows) if rows is not None \
        else rope_apply(q, pack["pos_ids"], rope_axes, base)
    k_r = rope_apply(k, pack["pos_ids"], rope_axes, base)
    if rows is not None:
        # attention needs every key of the sampled rows' samples, but only the
        # sampled query rows; scatter the roped query rows back in place.
        q_full = np.zeros(np.asarray(q).shape, dtype=np.float64)
        q_full[rows] = q_r
        q_r = q_full
    o, _ = varlen_attention(q_r, k_r, v, pack["cu_seqlens"], rows=rows)
    if rows is not None:
        y = gated_residual(np.asarray(x)[rows], o, mod, np.asarray(tok_sample)[rows],
                           np.asarray(tok_mod)[rows])
    else:
        y = gated_residual(x, o, mod, tok_sample, tok_mod)
    return x_mod, y, o


# ---------------------------------------------------------------------------
# Backward of the block  ([train]: the packed model is trained)
# ---------------------------------------------------------------------------
def gated_residual_bwd(dy, o, mod, tok_sample, tok_mod, S: int):
    """Gradients of ``y = x + gate[s, m] * O`` (chain rule, written out):
    dx = dy; dO = gate[s, m] * dy; dgate[s, m] = sum over the tokens t of sample
    s and modality m of dy[t] * O[t]. O and dO are viewed as [T][H*D]. Returns
    float64 (dx [T][hid], d_o [T][hid], dmod [S][2][3][hid] with only the GATE
    slot non-zero)."""
    dy = np.asarray(dy, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64).reshape(dy.shape[0], -1)
    tok_sample = np.asarray(tok_sample).astype(np.int64)
    tok_mod = np.asarray(tok_mod).astype(np.int64)
    gate = mod[tok_sample, tok_mod, GATE]
    dmod = np.zeros((S, 2, 3, dy.shape[1]), dtype=np.float64)
    np.add.at(dmod, (tok_sample, tok_mod, GATE), dy * o)
    return dy.copy(), gate * dy, dmod


def adaln_modulate_bwd(dxm, x, mod, tok_sample, tok_mod, S: int, eps: float = 1e-6):
    """Gradients of ``x_mod = xhat * (1 + scale[s, m]) + shift[s, m]`` with
    ``xhat = (x - mean) / sqrt(var + eps)`` over each row (population variance):
        dshift[s, m] = sum_t dx_mod[t],   dscale[s, m] = sum_t dx_mod[t] * xhat[t]
        g = dx_mod * (1 + scale)
        dx = (g - mean(g) - xhat * mean(g * xhat)) / sqrt(var + eps)
    (sums over the tokens of sample s and modality m; means over the row).
    Returns float64 (dx [T][hid], dmod [S][2][3][hid] with SHIFT and SCALE set)."""
    dxm = np.asarray(dxm, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    tok_sample = np.asarray(tok_sample).astype(np.int64)
    tok_mod = np.asarray(tok_mod).astype(np.int64)
    mu = x.mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(np.mean((x - mu) ** 2, axis=1, keepdims=True) + eps)
    xhat = (x - mu) * rstd
    scale = mod[tok_sample, tok_mod, SCALE]
    g = dxm * (1.0 + scale)
    dx = (g - g.mean(axis=1, keepdims=True) - xhat * (g * xhat).mean(axis=1, keepdims=True)) * rstd
    dmod = np.zeros((S, 2, 3, x.shape[1]), dtype=np.float64)
    np.add.at(dmod, (tok_sample, tok_mod, SHIFT), dxm)
    np.add.at(dmod, (tok_sample, tok_mod, SCALE), dxm * xhat)
    return dx, dmod


def rope_bwd(dx_r, pos_ids, rope_axes: int, base: float = 10000.0):
    """Gradient of ``rope_apply``: every pair rotation is orthogonal, so the
    gradient turns back by the same angle (the transpose):
    ``a = c dx0' + s dx1'``, ``b = -s dx0' + c dx1'``. [T][H][D] -> float64."""
    g = np.asarray(dx_r, dtype=np.float64)
    D = g.shape[-1]
    theta = rope_pair_angles(pos_ids, D, rope_axes, base)[:, None, :]
    cos, sin = np.cos(theta), np.sin(theta)
    g0, g1 = g[..., 0::2], g[..., 1::2]
    out = np.empty_like(g)
    out[..., 0::2] = g0 * cos + g1 * sin
    out[..., 1::2] = -g0 * sin + g1 * cos
    return out


def adaln_params_bwd(dmod, c, W):
    """Gradients of ``mod = c W`` (flattened to [S][6 hid]): dW = c^T dmod,
    dc = dmod W^T. Returns float64 (dc [S][C], dW [C][6 hid])."""
    c = np.asarray(c, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    dm = np.asarray(dmod, dtype=np.float64).reshape(c.shape[0], -1)
    return dm @ W.T, c.T @ dm


def block_bwd(dy, dx_mod, x, q, k, v, mod, pack, rope_axes: int, base: float = 10000.0,
              eps: float = 1e-6):
    """Backward of ``block_fwd`` for upstream gradients dy (of y) and dx_mod
    (of x_mod): the gate, the attention (from the rotated q, k), RoPE and the
    adaLN modulation in reverse order. Returns float64 (dx, dq, dk, dv, dmod);
    dmod [S][2][3][hid] holds the shift, scale and gate gradients."""
    S = len(pack["cu_seqlens"]) - 1
    tok_sample, tok_mod = pack["tok_sample"], pack["tok_mod"]
    q_r = rope_apply(q, pack["pos_ids"], rope_axes, base)
    k_r = rope_apply(k, pack["pos_ids"], rope_axes, base)
    o, _ = varlen_attention(q_r, k_r, v, pack["cu_seqlens"])
    dx_res, d_o, dmod_gate = gated_residual_bwd(dy, o, mod, tok_sample, tok_mod, S)
    T, H, D = np.asarray(q).shape
    dq_r, dk_r, dv = varlen_attention_bwd(q_r, k_r, v, d_o.reshape(T, H, D), pack["cu_seqlens"])
    dq = rope_bwd(dq_r, pack["pos_ids"], rope_axes, base)
    dk = rope_bwd(dk_r, pack["pos_ids"], rope_axes, base)
    dx_ln, dmod_ln = adaln_modulate_bwd(dx_mod, x, mod, tok_sample, tok_mod, S, eps)
    return dx_res + dx_ln, dq, dk, dv, dmod_gate + dmod_ln


# ---------------------------------------------------------------------------
# Modality-specific linear layer  ([norm])
# ---------------------------------------------------------------------------
def gelu_tanh(x) -> np.ndarray:
    """GELU in its tanh form, 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).

    Reading: the pages do not describe the MLP branch of the block; the form
    taken is the one DiT-family blocks use."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def modality_linear(x, W, tok_mod, act: str = "none") -> np.ndarray:
    """The per-modality projection of an MMDiT block.

    [norm]: the backbone is an MMDiT with modality-specific normalization and
    joint self-attention; in an MMDiT the image and the text stream also keep
    their own projection weights, and the joint attention runs on the
    concatenation. Reading (the pages give no layer shapes): one linear map per
    modality, no bias, ``out[t] = x[t] @ W[m(t)].T`` with m(t) = tok_mod[t]
    (0 image, 1 text) and W stored as [2][N][K] (out features, in features).

    x: [T][K]; act: "none" or "gelu" (gelu_tanh applied to every output);
    returns float64 [T][N].
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    tok_mod = np.asarray(tok_mod)
    out = np.zeros((x.shape[0], W.shape[1]), dtype=np.float64)
    for m in (MOD_IMG, MOD_TXT):
        sel = tok_mod == m
        out[sel] = x[sel] @ W[m].T
    if act == "gelu":
        out = gelu_tanh(out)
    elif act != "none":
        raise ValueError("act must be 'none' or 'gelu'")
    return out


# ---------------------------------------------------------------------------
# The whole MMDiT block around the joint-attention path  ([norm], [fuse])
# ---------------------------------------------------------------------------
def store_bf16(a) -> np.ndarray:
    """The bf16 value a block stores for an intermediate result (round to
    float32, then to bf16 nearest-even), back in float64."""
    from packgen import bf16_bits_to_f32, f32_to_bf16_bits
    return bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(a, dtype=np.float32))).astype(np.float64)


def mmdit_block_fwd(x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, pack, H: int, D: int,
                    rope_axes: int, base: float = 10000.0, eps: float = 1e-6, rows=None,
                    store=store_bf16):
    """One NR-MMDiT block forward over a pack.

    [norm]: modality-specific normalization and joint self-attention; [fuse]:
    adaptive normalization / RoPE / gating. Reading (the pages give the
    operations, not the block's wiring): the DiT-family block with two gated
    branches, each with its own modulation vectors (shift, scale, gate) per
    sample and modality, and modality-specific projections:
        x1 = adaLN(x; mod_attn)
        q, k, v = x1 Wq[m]^T, x1 Wk[m]^T, x1 Wv[m]^T       (per token modality m)
        o  = joint varlen attention of RoPE(q), RoPE(k), v  (per sample)
        y1 = x + gate_attn * (o Wo[m]^T)
        x2 = adaLN(y1; mod_mlp)
        y  = y1 + gate_mlp * (GELU(x2 Wup[m]^T) Wdown[m]^T)
    Every intermediate is stored in bf16 (``store``), as the GPU block stores
    them; the final y is returned unrounded (float64). ``rows`` restricts the
    output to those rows (keys and values are still computed for every row).
    """
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    ts, tm = np.asarray(pack["tok_sample"]), np.asarray(pack["tok_mod"])
    r = np.arange(T) if rows is None else np.asarray(rows)
    x1 = store(adaln_modulate(x, mod_attn, ts, tm, eps))
    k = store(modality_linear(x1, Wk, tm)).reshape(T, H, D)
    v = store(modality_linear(x1, Wv, tm)).reshape(T, H, D)
    q = np.zeros((T, H, D))
    q[r] = store(modality_linear(x1[r], Wq, tm[r])).reshape(-1, H, D)
    q_r = np.zeros((T, H, D))
    q_r[r] = store(rope_apply(q[r], np.asarray(pack["pos_ids"])[r], rope_axes, base))
    k_r = store(rope_apply(k, pack["pos_ids"], rope_axes, base))
    o, _ = varlen_attention(q_r, k_r, v, pack["cu_seqlens"], rows=r)
    o = store(o).reshape(len(r), H * D)
    a = store(modality_linear(o, Wo, tm[r]))
    y1 = store(gated_residual(x[r], a, mod_attn, ts[r], tm[r]))
    x2 = store(adaln_modulate(y1, mod_mlp, ts[r], tm[r], eps))
    h = store(modality_linear(x2, Wup, tm[r], "gelu"))
    mlp = store(modality_linear(h, Wdown, tm[r]))
    return gated_residual(y1, mlp, mod_mlp, ts[r], tm[r])


def gelu_tanh_bwd(z, dh) -> np.ndarray:
    """Gradient through ``gelu_tanh`` at pre-activation z: with
    u = sqrt(2/pi) (z + 0.044715 z^3),
    d gelu / dz = 0.5 (1 + tanh u) + 0.5 z (1 - tanh^2 u) sqrt(2/pi) (1 + 3 * 0.044715 z^2)."""
    z = np.asarray(z, dtype=np.float64)
    c = math.sqrt(2.0 / math.pi)
    th = np.tanh(c * (z + 0.044715 * z ** 3))
    return np.asarray(dh, dtype=np.float64) * (
        0.5 * (1.0 + th) + 0.5 * z * (1.0 - th * th) * c * (1.0 + 3.0 * 0.044715 * z * z))


def modality_linear_bwd(x, W, tok_mod, dout):
    """Gradients of ``out[t] = x[t] @ W[m(t)].T`` (no activation):
    dx[t] = dout[t] @ W[m(t)], dW[m] = sum over the tokens of modality m of
    dout[t]^T x[t]. Returns float64 (dx [T][K], dW [2][N][K])."""
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    tok_mod = np.asarray(tok_mod)
    dx = np.zeros_like(x)
    dW = np.zeros_like(W)
    for m in (MOD_IMG, MOD_TXT):
        sel = tok_mod == m
        dx[sel] = dout[sel] @ W[m]
        dW[m] = dout[sel].T @ x[sel]
    return dx, dW


def mmdit_block_bwd(dy, x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, pack, H: int, D: int,
                    rope_axes: int, base: float = 10000.0, eps: float = 1e-6):
    """Backward of ``mmdit_block_fwd`` without intermediate rounding (every
    intermediate kept in float64), for the upstream gradient dy of y: the MLP
    branch (gate, down projection, GELU, up projection, adaLN), then the
    attention branch (gate, output projection, attention, RoPE, the three input
    projections, adaLN), the residual path carrying dy through both. Returns a
    dict of float64 gradients: x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    S = len(pack["cu_seqlens"]) - 1
    ts, tm = np.asarray(pack["tok_sample"]), np.asarray(pack["tok_mod"])
    # forward, keeping what the backward needs
    x1 = adaln_modulate(x, mod_attn, ts, tm, eps)
    q = modality_linear(x1, Wq, tm).reshape(T, H, D)
    k = modality_linear(x1, Wk, tm).reshape(T, H, D)
    v = modality_linear(x1, Wv, tm).reshape(T, H, D)
    q_r = rope_apply(q, pack["pos_ids"], rope_axes, base)
    k_r = rope_apply(k, pack["pos_ids"], rope_axes, base)
    o, _ = varlen_attention(q_r, k_r, v, pack["cu_seqlens"])
    o = o.reshape(T, H * D)
    a = modality_linear(o, Wo, tm)
    y1 = gated_residual(x, a, mod_attn, ts, tm)
    x2 = adaln_modulate(y1, mod_mlp, ts, tm, eps)
    z = modality_linear(x2, Wup, tm)
    h = gelu_tanh(z)
    mlp = modality_linear(h, Wdown, tm)
    # MLP branch
    dy1, dmlp, dmod_mlp = gated_residual_bwd(dy, mlp, mod_mlp, ts, tm, S)
    dh, dWdown = modality_linear_bwd(h, Wdown, tm, dmlp)
    dx2, dWup = modality_linear_bwd(x2, Wup, tm, gelu_tanh_bwd(z, dh))
    dy1_ln, dmod_mlp_ln = adaln_modulate_bwd(dx2, y1, mod_mlp, ts, tm, S, eps)
    dy1 = dy1 + dy1_ln
    dmod_mlp = dmod_mlp + dmod_mlp_ln
    # attention branch
    dx, da, dmod_attn = gated_residual_bwd(dy1, a, mod_attn, ts, tm, S)
    do, dWo = modality_linear_bwd(o, Wo, tm, da)
    dq_r, dk_r, dv = varlen_attention_bwd(q_r, k_r, v, do.reshape(T, H, D), pack["cu_seqlens"])
    dq = rope_bwd(dq_r, pack["pos_ids"], rope_axes, base).reshape(T, H * D)
    dk = rope_bwd(dk_r, pack["pos_ids"], rope_axes, base).reshape(T, H * D)
    dx1q, dWq = modality_linear_bwd(x1, Wq, tm, dq)
    dx1k, dWk = modality_linear_bwd(x1, Wk, tm, dk)
    dx1v, dWv = modality_linear_bwd(x1, Wv, tm, dv.reshape(T, H * D))
    dx_ln, dmod_attn_ln = adaln_modulate_bwd(dx1q + dx1k + dx1v, x, mod_attn, ts, tm, S, eps)
    return dict(x=dx + dx_ln, Wq=dWq, Wk=dWk, Wv=dWv, Wo=dWo, Wup=dWup, Wdown=dWdown,
                mod_attn=dmod_attn + dmod_attn_ln, mod_mlp=dmod_mlp)


# ---------------------------------------------------------------------------
# Packed classifier-free guidance  ([cfg])
# ---------------------------------------------------------------------------
def cfg_combine(v, descs: Sequence, pairs: Sequence, w: float) -> np.ndarray:
    """Classifier-free guidance over a packed-CFG pack.

    [cfg]: the conditional and the unconditional branch of an image run as two
    samples of one pack, in a single forward. The pages do not give the
    combine; the reading taken is the usual classifier-free guidance form,
    applied to the image tokens of each (conditional, unconditional) pair:
    ``out = v_u + w * (v_c - v_u)``, where row i of a pair's output takes row i
    of each sample's image tokens (a sample's image tokens come first, see
    ``pack_build``). Both samples of a pair must have the same number of image
    tokens; their text tokens (prompt vs. empty prompt) are not part of it.

    v: [T][C] per-token outputs of the pack; pairs: (cond, uncond) sample
    indices. Returns float64 [sum of the pairs' image-token counts][C], pairs in
    the order given.
    """
    v = np.asarray(v, dtype=np.float64)
    rows = [tuple(d.as_tuple()) if hasattr(d, "as_tuple") else tuple(d) for d in descs]
    n_tok = [F * Hg * Wg + L for (F, Hg, Wg, L, *_r) in rows]
    n_img = [F * Hg * Wg for (F, Hg, Wg, _L, *_r) in rows]
    cu = np.concatenate([[0], np.cumsum(n_tok)]).astype(np.int64)
    if v.shape[0] != cu[-1]:
        raise ValueError("v has the wrong number of rows for the pack")
    out = []
    for (c, u) in pairs:
        if not (0 <= c < len(rows) and 0 <= u < len(rows)) or c == u:
            raise ValueError("bad pair")
        if n_img[c] != n_img[u]:
            raise ValueError("the two branches of a pair need the same image grid")
        n = n_img[c]
        v_c = v[cu[c]:cu[c] + n]
        v_u = v[cu[u]:cu[u] + n]
        out.append(v_u + w * (v_c - v_u))
    C = v.shape[1] if v.ndim == 2 else 0
    return np.concatenate(out, axis=0) if out else np.zeros((0, C))


def useful_attention_flops(descs: Sequence, H: int, D: int) -> float:
    """Useful attention FLOPs of a pack: ``4 * D * H * sum n_s^2`` over the real
    samples (QK^T and PV, 2 FLOPs per multiply-add, only within-sample pairs,
    the padding segment excluded)."""
    tot = 0
    for d in descs:
        t = tuple(d.as_tuple()) if hasattr(d, "as_tuple") else tuple(d)
        F, Hg, Wg, L = t[:4]
        dummy = t[4] if len(t) > 4 else 0
        if dummy:
            continue
        n = F * Hg * Wg + L
        tot += n * n
    return 4.0 * D * H * tot
