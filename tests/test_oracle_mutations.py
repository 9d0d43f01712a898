"""Plant plausible mistakes in copies of the oracle (on the CPU) and check
that the pins catch each one. A pin set that passes a broken oracle would not
be evidence of anything."""

import math

import numpy as np
import pytest

import oracle
from oracle import mf_oracle as mo
import pins


def _rope_sign_flip(x, pos_ids, rope_axes, base=10000.0, rows=None):
    x = np.asarray(x, dtype=np.float64)
    th = mo.rope_pair_angles(np.asarray(pos_ids), x.shape[-1], rope_axes, base)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = x[..., 0::2] * np.cos(th) + x[..., 1::2] * np.sin(th)   # wrong sign
    out[..., 1::2] = x[..., 0::2] * np.sin(th) + x[..., 1::2] * np.cos(th)
    return out


def _rope_half_split(x, pos_ids, rope_axes, base=10000.0, rows=None):
    # pairs (i, i + D/2) instead of adjacent channels
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    th = mo.rope_pair_angles(np.asarray(pos_ids), D, rope_axes, base)[:, None, :]
    a, b = x[..., :D // 2], x[..., D // 2:]
    return np.concatenate([a * np.cos(th) - b * np.sin(th), a * np.sin(th) + b * np.cos(th)], -1)


def _rope_axes_swapped(x, pos_ids, rope_axes, base=10000.0, rows=None):
    p = np.asarray(pos_ids).copy()
    p[:, [1, 2]] = p[:, [2, 1]]
    return mo.rope_apply(x, p, rope_axes, base)


def _mod_shift_scale_swapped(c, W, hid):
    m = mo.adaln_params(c, W, hid)
    return m[:, :, [1, 0, 2], :]


def _ln_sample_var(x, eps):
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = np.var(x, axis=-1, ddof=1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def _attention_ignores_pack(q, k, v, cu_seqlens, scale=None, rows=None, chunk=2048):
    T = np.asarray(q).shape[0]
    return mo.varlen_attention(q, k, v, [0, T], scale, rows, chunk)


def _attention_no_scale(q, k, v, cu_seqlens, scale=None, rows=None, chunk=2048):
    return mo.varlen_attention(q, k, v, cu_seqlens, 1.0, rows, chunk)


def _attention_transposed_pv(q, k, v, cu_seqlens, scale=None, rows=None, chunk=2048):
    # uses the key matrix instead of the value matrix (an operand mix-up)
    return mo.varlen_attention(q, k, k, cu_seqlens, scale, rows, chunk)


def _pack_text_from_zero(descs, rope_axes):
    p = mo.pack_build(descs, rope_axes)
    pos = p["pos_ids"].copy()
    cu = p["cu_seqlens"]
    for s, d in enumerate(descs):
        F, Hg, Wg, L = d.as_tuple()[:4] if hasattr(d, "as_tuple") else d[:4]
        n_img = F * Hg * Wg
        pos[cu[s] + n_img:cu[s + 1], :] = np.arange(L)[:, None]
    p["pos_ids"] = pos
    return p


def _pack_col_major(descs, rope_axes):
    p = mo.pack_build(descs, rope_axes)
    pos = p["pos_ids"].copy()
    cu = p["cu_seqlens"]
    for s, d in enumerate(descs):
        F, Hg, Wg, L = d.as_tuple()[:4] if hasattr(d, "as_tuple") else d[:4]
        f, w, h = np.meshgrid(np.arange(F), np.arange(Wg), np.arange(Hg), indexing="ij")
        n_img = F * Hg * Wg
        pos[cu[s]:cu[s] + n_img] = np.stack([f.ravel(), h.ravel(), w.ravel()], 1)
    p["pos_ids"] = pos
    return p


def _gate_uses_scale(x, o, mod, tok_sample, tok_mod, rows=None):
    m = mod[:, :, [0, 1, 1], :]
    return mo.gated_residual(x, o, m, tok_sample, tok_mod, rows)


def _cfg_branches_swapped(v, descs, pairs, w):
    return mo.cfg_combine(v, descs, [(u, c) for (c, u) in pairs], w)


def _cfg_text_rows(v, descs, pairs, w):
    # takes the pair's rows from the end of each sample (its text tokens) instead
    rows = [tuple(d) for d in descs]
    n = [F * H * W + L for (F, H, W, L, *_r) in rows]
    cu = np.concatenate([[0], np.cumsum(n)])
    out = []
    for (c, u) in pairs:
        k = rows[c][0] * rows[c][1] * rows[c][2]
        vc = np.asarray(v, dtype=np.float64)[cu[c + 1] - k:cu[c + 1]]
        vu = np.asarray(v, dtype=np.float64)[cu[u + 1] - k:cu[u + 1]]
        out.append(vu + w * (vc - vu))
    return np.concatenate(out)


def _linear_modality_swapped(x, W, tok_mod):
    return mo.modality_linear(x, np.asarray(W)[::-1], tok_mod)


def _linear_untransposed(x, W, tok_mod):
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    out = np.zeros((x.shape[0], W.shape[1]))
    for m in (0, 1):
        sel = np.asarray(tok_mod) == m
        out[sel] = x[sel][:, :W.shape[1]] @ W[m][:, :W.shape[1]]  # W used as [K][N]
    return out


def _gelu_sigmoid_form(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-1.702 * x))  # another approximation, not this one


def _gelu_no_cubic(x):
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * x))


def _mmdit_gelu_after_down(x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, pack, H, D,
                           rope_axes, base=10000.0, eps=1e-6, rows=None, store=mo.store_bf16):
    # the activation after the second MLP layer instead of between the two
    full = mo.mmdit_block_fwd(x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, pack, H, D,
                                   rope_axes, base, eps, rows, store)
    y1 = mo.mmdit_block_fwd(x, Wq, Wk, Wv, Wo, Wup, np.zeros_like(Wdown), mod_attn, mod_mlp, pack,
                            H, D, rope_axes, base, eps, rows, store)
    gate = np.asarray(mod_mlp)[pack["tok_sample"], pack["tok_mod"], 2]
    branch = (full - y1) / np.where(gate == 0, 1.0, gate)
    return y1 + gate * mo.gelu_tanh(branch)


def _mmdit_mlp_uses_attn_mod(x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, pack, H, D,
                             rope_axes, base=10000.0, eps=1e-6, rows=None, store=mo.store_bf16):
    return mo.mmdit_block_fwd(x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_attn, pack, H, D,
                              rope_axes, base, eps, rows, store)


def _attn_bwd_no_delta(q, k, v, d_o, cu_seqlens, scale=None):
    # the softmax Jacobian without its rowsum(dO * O) term
    q, k, v, d_o = (np.asarray(a, dtype=np.float64) for a in (q, k, v, d_o))
    cu = np.asarray(cu_seqlens)
    dq, dk, dv = (np.zeros_like(q) for _ in range(3))
    sc = 1.0 / math.sqrt(q.shape[2])
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        if hi == lo:
            continue
        for h in range(q.shape[1]):
            S = q[lo:hi, h] @ k[lo:hi, h].T * sc
            P = np.exp(S - S.max(1, keepdims=True))
            P /= P.sum(1, keepdims=True)
            dv[lo:hi, h] = P.T @ d_o[lo:hi, h]
            dS = P * (d_o[lo:hi, h] @ v[lo:hi, h].T)
            dq[lo:hi, h] = sc * dS @ k[lo:hi, h]
            dk[lo:hi, h] = sc * dS.T @ q[lo:hi, h]
    return dq, dk, dv


def _attn_bwd_unscaled_dk(q, k, v, d_o, cu_seqlens, scale=None):
    dq, dk, dv = mo.varlen_attention_bwd(q, k, v, d_o, cu_seqlens, scale)
    return dq, dk * math.sqrt(np.asarray(q).shape[2]), dv


def _adaln_bwd_no_xhat_term(dxm, x, mod, tok_sample, tok_mod, S, eps=1e-6):
    # the LayerNorm gradient without its xhat * mean(g * xhat) projection
    x = np.asarray(x, dtype=np.float64)
    dxm = np.asarray(dxm, dtype=np.float64)
    ts, tm = np.asarray(tok_sample).astype(np.int64), np.asarray(tok_mod).astype(np.int64)
    mu = x.mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(np.mean((x - mu) ** 2, axis=1, keepdims=True) + eps)
    g = dxm * (1.0 + mod[ts, tm, 1])
    _, dmod = mo.adaln_modulate_bwd(dxm, x, mod, tok_sample, tok_mod, S, eps)
    return (g - g.mean(axis=1, keepdims=True)) * rstd, dmod


def _adaln_bwd_scale_ignored(dxm, x, mod, tok_sample, tok_mod, S, eps=1e-6):
    # dx computed as if scale were 0
    dx, dmod = mo.adaln_modulate_bwd(dxm, x, np.zeros_like(mod), tok_sample, tok_mod, S, eps)
    _, dmod = mo.adaln_modulate_bwd(dxm, x, mod, tok_sample, tok_mod, S, eps)
    return dx, dmod


def _rope_bwd_forward_rotation(dx_r, pos_ids, rope_axes, base=10000.0):
    # turns the gradient forwards instead of back
    return mo.rope_apply(dx_r, pos_ids, rope_axes, base)


def _block_bwd_sample_blind_gate(dy, dx_mod, x, q, k, v, mod, pack, rope_axes, base=10000.0,
                                 eps=1e-6):
    # every sample's gate gradient summed into sample 0
    dx, dq, dk, dv, dmod = mo.block_bwd(dy, dx_mod, x, q, k, v, mod, pack, rope_axes, base, eps)
    dmod = dmod.copy()
    dmod[0, :, 2] = dmod[:, :, 2].sum(axis=0)
    dmod[1:, :, 2] = 0.0
    return dx, dq, dk, dv, dmod


def _block_bwd_no_residual(dy, dx_mod, x, q, k, v, mod, pack, rope_axes, base=10000.0,
                           eps=1e-6):
    # dx loses the identity path of y = x + gate * O
    dx, dq, dk, dv, dmod = mo.block_bwd(dy, dx_mod, x, q, k, v, mod, pack, rope_axes, base, eps)
    return dx - np.asarray(dy, dtype=np.float64), dq, dk, dv, dmod


def _gelu_bwd_no_sech_term(z, dh):
    # keeps 0.5 (1 + tanh u), drops the z * sech^2 part
    z = np.asarray(z, dtype=np.float64)
    th = np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3))
    return np.asarray(dh, dtype=np.float64) * 0.5 * (1.0 + th)


def _mmdit_bwd_swapped_weight_grads(*args, **kwargs):
    # the image and text gradients of the up projection land in each other's slot
    g = mo.mmdit_block_bwd(*args, **kwargs)
    g = dict(g)
    g["Wup"] = g["Wup"][::-1].copy()
    return g


def _mmdit_bwd_no_mlp_norm_path(dy, x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, pack, H, D,
                                rope_axes, base=10000.0, eps=1e-6):
    # the attention branch sees only the identity path of the MLP branch
    saved = mo.adaln_modulate_bwd
    calls = []

    def zero_first(*a, **k):
        dx, dmod = saved(*a, **k)
        if not calls:
            calls.append(1)
            dx = np.zeros_like(dx)
        return dx, dmod

    mo.adaln_modulate_bwd = zero_first
    try:
        return mo.mmdit_block_bwd(dy, x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, pack, H,
                                  D, rope_axes, base, eps)
    finally:
        mo.adaln_modulate_bwd = saved


MUTANTS = [
    ("rope sign flip", lambda: pins.check_rope_relative(_rope_sign_flip) or
     pins.check_rope_textbook_1d(_rope_sign_flip)),
    ("rope half-split pairs", lambda: pins.check_rope_textbook_1d(_rope_half_split)),
    ("rope h/w swapped", lambda: pins.check_rope_textbook_1d(_rope_axes_swapped)),
    ("shift/scale swapped", lambda: pins.check_mod_layout(_mod_shift_scale_swapped)),
    ("LN sample variance", lambda: pins.check_layernorm_moments(_ln_sample_var)),
    ("attention across samples", lambda: pins.check_attention_vs_sdpa(_attention_ignores_pack)),
    ("attention without 1/sqrt(D)", lambda: pins.check_attention_vs_sdpa(_attention_no_scale)),
    ("K used as V", lambda: pins.check_attention_vs_brute(_attention_transposed_pv)),
    ("text positions from 0", lambda: pins.check_pack_tiny_closed_form(_pack_text_from_zero)),
    ("column-major grid", lambda: pins.check_pack_tiny_closed_form(_pack_col_major)),
    ("gate reads scale", lambda: pins.check_gate(_gate_uses_scale, oracle.adaln_params,
                                                 oracle.pack_build)),
    ("CFG branches swapped", lambda: pins.check_cfg_special_weights(_cfg_branches_swapped)),
    ("CFG rows from the text end", lambda: pins.check_cfg_row_map(_cfg_text_rows)),
    ("linear weights of the other modality",
     lambda: pins.check_linear_routing(_linear_modality_swapped)),
    ("linear weight not transposed", lambda: pins.check_linear_vs_brute(_linear_untransposed)),
    ("GELU sigmoid form", lambda: pins.check_gelu(_gelu_sigmoid_form)),
    ("GELU without the cubic term", lambda: pins.check_gelu(_gelu_no_cubic)),
    ("block: GELU after the down projection",
     lambda: pins.check_mmdit_vs_brute(_mmdit_gelu_after_down, oracle.pack_build)),
    ("attention backward without the rowsum term",
     lambda: pins.check_attention_bwd_vs_autograd(_attn_bwd_no_delta)),
    ("attention backward without the rowsum term, against the scalar loops",
     lambda: pins.check_attention_bwd_vs_brute(_attn_bwd_no_delta)),
    ("attention backward dK without the scale",
     lambda: pins.check_attention_bwd_finite_diff(_attn_bwd_unscaled_dk, oracle.varlen_attention)),
    ("adaLN backward without the xhat projection",
     lambda: pins.check_adaln_bwd_vs_torch_layer_norm(_adaln_bwd_no_xhat_term)),
    ("adaLN backward ignoring the scale",
     lambda: pins.check_adaln_bwd_vs_torch_layer_norm(_adaln_bwd_scale_ignored)),
    ("RoPE backward turning forwards",
     lambda: pins.check_rope_bwd_adjoint(_rope_bwd_forward_rotation, oracle.rope_apply)),
    ("block backward with the gate gradient blind to samples",
     lambda: pins.check_block_bwd_finite_diff(_block_bwd_sample_blind_gate, oracle.block_fwd)),
    ("block backward without the residual path",
     lambda: pins.check_block_bwd_finite_diff(_block_bwd_no_residual, oracle.block_fwd)),
    ("GELU backward without the sech^2 term",
     lambda: pins.check_gelu_bwd_vs_torch(_gelu_bwd_no_sech_term)),
    ("MMDiT backward with image and text weight gradients swapped",
     lambda: pins.check_mmdit_bwd_finite_diff(_mmdit_bwd_swapped_weight_grads,
                                              oracle.mmdit_block_fwd)),
    ("MMDiT backward without the MLP branch's normalization path",
     lambda: pins.check_mmdit_bwd_finite_diff(_mmdit_bwd_no_mlp_norm_path,
                                              oracle.mmdit_block_fwd)),
    ("block: MLP branch modulated by the attention vectors",
     lambda: pins.check_mmdit_branch_gates(_mmdit_mlp_uses_attn_mod, oracle.pack_build)),
]


@pytest.mark.parametrize("name,run", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, run):
    with pytest.raises(AssertionError):
        run()
