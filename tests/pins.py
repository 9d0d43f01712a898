"""Reusable pin checks for the oracle.

Each ``check_*`` takes the oracle function(s) it pins as arguments and raises
AssertionError when they break a property fixed by the pages, by mathematics or
by an independent computation. ``test_oracle_pins.py`` runs them on the oracle;
``test_oracle_mutations.py`` runs them on deliberately broken copies to show
that each plausible slip is caught.
"""

from __future__ import annotations

import math

import numpy as np
import torch

from oracle import brute
from packgen import SampleDesc, make_random_pack


# --------------------------------------------------------------------- pack
def check_pack_vs_brute(pack_build):
    for seed in range(6):
        for axes in (2, 3):
            w = make_random_pack(100 + seed, S=1 + seed % 4, H=1, D=8, rope_axes=axes)
            p = pack_build(w.descs, axes)
            cu, pos, ts, tm = brute.brute_pack(w.descs, axes)
            assert p["cu_seqlens"].tolist() == cu
            assert p["pos_ids"].tolist() == [list(t) for t in pos]
            assert p["tok_sample"].tolist() == ts
            assert p["tok_mod"].tolist() == tm


def check_pack_tiny_closed_form(pack_build):
    # The 544-token pack: sample A = 16x16 grid + 20 text, B = 8x32 grid + 12 text.
    p = pack_build([SampleDesc(1, 16, 16, 20), SampleDesc(1, 8, 32, 12)], 2)
    nA, nB = 16 * 16 + 20, 8 * 32 + 12
    assert p["cu_seqlens"].tolist() == [0, nA, nA + nB]
    pos = p["pos_ids"]
    assert pos[0].tolist() == [0, 0, 0]
    assert pos[17].tolist() == [0, 1, 1]          # row-major: 17 = 1*16 + 1
    assert pos[255].tolist() == [0, 15, 15]
    assert pos[256].tolist() == [16, 16, 16]      # first text token: max(16,16) + 0
    assert pos[nA - 1].tolist() == [16 + 19] * 3
    assert pos[nA + 31].tolist() == [0, 0, 31]    # B is 8 rows of 32
    assert pos[nA + 32].tolist() == [0, 1, 0]
    assert pos[nA + 256].tolist() == [32, 32, 32]  # max(8,32) + 0
    assert int((p["tok_mod"] == 1).sum()) == 32
    assert p["tok_sample"][nA - 1] == 0 and p["tok_sample"][nA] == 1


def check_pack_edit_frames(pack_build):
    # Edit pack: source (f=0) and target (f=1) share every (h, w) ([edit]).
    p = pack_build([SampleDesc(2, 3, 4, 2)], 3)
    pos = p["pos_ids"]
    n_grid = 3 * 4
    assert (pos[:n_grid, 0] == 0).all() and (pos[n_grid:2 * n_grid, 0] == 1).all()
    assert (pos[:n_grid, 1:] == pos[n_grid:2 * n_grid, 1:]).all()
    assert pos[2 * n_grid].tolist() == [4, 4, 4]


# ---------------------------------------------------------------------- adaLN
def check_mod_layout(adaln_params):
    # W is a selector: column (3m + j)*hid + i reads conditioning entry
    # code(m, j, i) = (7m + 3j + 5i) mod C, so each slot has a distinct source.
    C, hid, S = 16, 5, 2
    c = np.arange(S * C, dtype=np.float64).reshape(S, C) + 1.0
    W = np.zeros((C, 6 * hid))
    for m in range(2):
        for j in range(3):
            for i in range(hid):
                W[(7 * m + 3 * j + 5 * i) % C, (3 * m + j) * hid + i] = 1.0
    mod = adaln_params(c, W, hid)
    assert mod.shape == (S, 2, 3, hid)
    for s in range(S):
        for m in range(2):
            for j in range(3):
                for i in range(hid):
                    assert mod[s, m, j, i] == c[s, (7 * m + 3 * j + 5 * i) % C]


def check_mod_vs_brute(adaln_params):
    rng = np.random.default_rng(7)
    c = rng.standard_normal((3, 6))
    W = rng.standard_normal((6, 6 * 4))
    got = adaln_params(c, W, 4)
    ref = brute.brute_mod(c.tolist(), W.tolist(), 4)
    assert np.allclose(got, np.array(ref), rtol=0, atol=1e-12)


def check_layernorm_moments(layer_norm_rows):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((20, 96)) * 3.0 + 1.5
    eps = 1e-6
    y = layer_norm_rows(x, eps)
    var = x.var(axis=1)
    assert np.allclose(y.mean(axis=1), 0.0, atol=1e-12)
    # population variance of the output is var / (var + eps)
    assert np.allclose(y.var(axis=1), var / (var + eps), atol=1e-12)
    # a constant row maps to zero (0 / sqrt(eps))
    assert np.allclose(layer_norm_rows(np.full((1, 8), 4.0), eps), 0.0)


def check_adaln_zero_map(adaln_params, adaln_modulate, layer_norm_rows, gated_residual):
    w = make_random_pack(11, S=3, H=2, D=8, rope_axes=2)
    from oracle import pack_build  # descriptors -> per-token ids
    p = pack_build(w.descs, 2)
    mod = adaln_params(w.c, np.zeros_like(w.W), w.hid)
    x = w.f32("x")
    assert np.array_equal(adaln_modulate(x, mod, p["tok_sample"], p["tok_mod"], 1e-6),
                          layer_norm_rows(x, 1e-6))
    o = np.random.default_rng(0).standard_normal((w.T, w.H, w.D))
    assert np.array_equal(gated_residual(x, o, mod, p["tok_sample"], p["tok_mod"]),
                          x.astype(np.float64))


def check_adaln_vs_brute(adaln_params, adaln_modulate, pack_build):
    w = make_random_pack(12, S=3, H=2, D=8, rope_axes=2)
    p = pack_build(w.descs, 2)
    mod = adaln_params(w.c, w.W, w.hid)
    x = w.f32("x")
    got = adaln_modulate(x, mod, p["tok_sample"], p["tok_mod"], 1e-6)
    for t in range(w.T):
        s, m = int(p["tok_sample"][t]), int(p["tok_mod"][t])
        ref = brute.brute_adaln_row(x[t].tolist(), mod[s, m, 0].tolist(), mod[s, m, 1].tolist(), 1e-6)
        assert np.allclose(got[t], ref, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------- RoPE
def _pos_rows(n, rng, hi=50):
    return rng.integers(0, hi, size=(n, 3)).astype(np.int32)


def check_rope_identity_and_norm(rope_apply):
    rng = np.random.default_rng(5)
    for D, axes in ((64, 2), (128, 2), (128, 3), (8, 2)):
        x = rng.standard_normal((9, 3, D))
        assert np.array_equal(rope_apply(x, np.zeros((9, 3), np.int32), axes), x)
        y = rope_apply(x, _pos_rows(9, rng), axes)
        n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
        n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
        assert np.allclose(n0, n1, rtol=1e-12, atol=1e-12)


def check_rope_relative(rope_apply):
    """<R(p) q, R(p') k> depends only on p - p' on every axis."""
    rng = np.random.default_rng(6)
    for D, axes in ((64, 2), (128, 2), (128, 3)):
        q = rng.standard_normal((1, 1, D))
        k = rng.standard_normal((1, 1, D))
        for _ in range(5):
            p = _pos_rows(1, rng)
            pp = _pos_rows(1, rng)
            shift = rng.integers(0, 30, size=(1, 3)).astype(np.int32)
            a = np.sum(rope_apply(q, p, axes) * rope_apply(k, pp, axes))
            b = np.sum(rope_apply(q, p + shift, axes) * rope_apply(k, pp + shift, axes))
            assert abs(a - b) < 1e-9 * max(1.0, abs(a))
        # and it does depend on the difference on each rotated axis
        p = np.zeros((1, 3), np.int32)
        comps = (1, 2) if axes == 2 else (0, 1, 2)
        base_val = np.sum(rope_apply(q, p, axes) * rope_apply(k, p, axes))
        for comp in comps:
            pp = p.copy()
            pp[0, comp] = 3
            moved = np.sum(rope_apply(q, p, axes) * rope_apply(k, pp, axes))
            assert abs(moved - base_val) > 1e-6


def check_rope_textbook_1d(rope_apply):
    """A 2D pack whose grid is one column wide (w = 0 everywhere) reduces to
    textbook 1D RoPE on the h channels, written here as complex multiplication
    z_i * exp(i * p * base**(-2i/d)) over the first d = D/2 channels, while the
    w channels stay put."""
    rng = np.random.default_rng(8)
    for D in (64, 128):
        d = D // 2
        x = rng.standard_normal((7, 2, D))
        h = np.arange(7)
        pos = np.stack([np.zeros(7), h, np.zeros(7)], axis=1).astype(np.int32)
        y = rope_apply(x, pos, 2)
        z = x[..., 0:d:2] + 1j * x[..., 1:d:2]
        omega = 10000.0 ** (-np.arange(d // 2) * 2.0 / d)
        zr = z * np.exp(1j * h[:, None, None] * omega[None, None, :])
        assert np.allclose(y[..., 0:d:2], zr.real, atol=1e-12)
        assert np.allclose(y[..., 1:d:2], zr.imag, atol=1e-12)
        assert np.array_equal(y[..., d:], x[..., d:])


def check_rope_3d_layout(rope_apply):
    """3D, D = 128: chunks of 42 channels for f, h, w; channels 126-127 are
    never rotated; moving only the frame index touches only channels 0-41."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((4, 1, 128))
    base_pos = np.array([[0, 5, 7]] * 4, np.int32)
    y0 = rope_apply(x, base_pos, 3)
    pos_f = base_pos.copy()
    pos_f[:, 0] = 1
    y1 = rope_apply(x, pos_f, 3)
    assert np.array_equal(y0[..., 42:], y1[..., 42:])
    assert not np.allclose(y0[..., :42], y1[..., :42])
    far = np.array([[9, 99, 999]] * 4, np.int32)
    assert np.array_equal(rope_apply(x, far, 3)[..., 126:], x[..., 126:])
    # angle of pair i of the h chunk at h = 1, recovered with atan2 from a unit pair
    e = np.zeros((1, 1, 128))
    e[..., 42::2] = 1.0  # the first channel of every pair from channel 42 on
    ang = rope_apply(e, np.array([[0, 1, 0]], np.int32), 3)
    got = np.arctan2(ang[0, 0, 43:84:2], ang[0, 0, 42:84:2])
    assert np.allclose(got, 10000.0 ** (-np.arange(21) * 2.0 / 42), atol=1e-12)


def check_rope_vs_brute(rope_apply, pack_build):
    for axes in (2, 3):
        w = make_random_pack(13 + axes, S=3, H=2, D=16, rope_axes=axes)
        p = pack_build(w.descs, axes)
        q = w.f32("q")
        got = rope_apply(q, p["pos_ids"], axes)
        for t in range(w.T):
            for h in range(w.H):
                ref = brute.brute_rope_vec(q[t, h].tolist(), p["pos_ids"][t].tolist(), axes)
                assert np.allclose(got[t, h], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------------ attention
def _sdpa64(q, k, v):
    """torch SDPA in float64 on CPU for one sample: q,k,v [n][H][D]."""
    tq = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2)))[None]
    tk = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))[None]
    tv = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))[None]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    return o[0].numpy().transpose(1, 0, 2)


def check_attention_vs_sdpa(varlen_attention):
    rng = np.random.default_rng(20)
    # a single-sample pack is ordinary full attention
    for n, H, D in ((1, 1, 8), (37, 2, 64), (300, 3, 128)):
        q, k, v = (rng.standard_normal((n, H, D)) for _ in range(3))
        o, _ = varlen_attention(q, k, v, [0, n])
        assert np.allclose(o, _sdpa64(q, k, v), rtol=1e-10, atol=1e-12)
    # a pack is block-diagonal: each sample equals attention over itself alone
    lens = [5, 130, 1, 64]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, D = int(cu[-1]), 2, 16
    q, k, v = (rng.standard_normal((T, H, D)) for _ in range(3))
    o, _ = varlen_attention(q, k, v, cu)
    for s in range(len(lens)):
        lo, hi = cu[s], cu[s + 1]
        assert np.allclose(o[lo:hi], _sdpa64(q[lo:hi], k[lo:hi], v[lo:hi]), rtol=1e-10, atol=1e-12)


def check_attention_lse(varlen_attention):
    from scipy.special import logsumexp
    rng = np.random.default_rng(21)
    lens = [3, 40]
    cu = [0, 3, 43]
    q, k, v = (rng.standard_normal((43, 2, 8)) for _ in range(3))
    _, lse = varlen_attention(q, k, v, cu)
    for s in range(2):
        for h in range(2):
            sc = q[cu[s]:cu[s + 1], h] @ k[cu[s]:cu[s + 1], h].T / math.sqrt(8)
            assert np.allclose(lse[h, cu[s]:cu[s + 1]], logsumexp(sc, axis=1), atol=1e-12)
    assert len(lens) == 2


def check_attention_permutation(varlen_attention):
    """Reordering the samples of a pack reorders the outputs, bit for bit."""
    rng = np.random.default_rng(22)
    lens = [7, 19, 3, 11]
    H, D = 2, 8
    segs = [tuple(rng.standard_normal((n, H, D)) for _ in range(3)) for n in lens]

    def run(order):
        q = np.concatenate([segs[i][0] for i in order])
        k = np.concatenate([segs[i][1] for i in order])
        v = np.concatenate([segs[i][2] for i in order])
        cu = np.concatenate([[0], np.cumsum([lens[i] for i in order])])
        o, _ = varlen_attention(q, k, v, cu)
        return [o[cu[j]:cu[j + 1]] for j in range(len(order))]

    ref = run([0, 1, 2, 3])
    perm = [2, 0, 3, 1]
    got = run(perm)
    for j, i in enumerate(perm):
        assert np.array_equal(got[j], ref[i])


def check_attention_equal_v(varlen_attention):
    """If every key of a sample carries the same value vector, every query of
    that sample returns it (softmax weights sum to one)."""
    rng = np.random.default_rng(23)
    cu = [0, 4, 50, 51]
    T, H, D = 51, 2, 8
    q = rng.standard_normal((T, H, D)) * 4
    k = rng.standard_normal((T, H, D)) * 4
    v = np.zeros((T, H, D))
    for s in range(3):
        v[cu[s]:cu[s + 1]] = rng.standard_normal((1, H, D))
    o, _ = varlen_attention(q, k, v, cu)
    assert np.allclose(o, v, rtol=0, atol=1e-12)


def check_attention_vs_brute(varlen_attention):
    for seed, D in ((30, 8), (31, 64), (32, 8)):
        rng = np.random.default_rng(seed)
        lens = [int(x) for x in rng.integers(1, 41, size=int(rng.integers(1, 4)))]
        H = int(rng.integers(1, 3))
        cu = [0]
        for n in lens:
            cu.append(cu[-1] + n)
        T = cu[-1]
        q, k, v = (rng.standard_normal((T, H, D)) for _ in range(3))
        o, _ = varlen_attention(q, k, v, cu)
        ref = brute.brute_attention(q.tolist(), k.tolist(), v.tolist(), cu)
        assert np.allclose(o, np.array(ref), rtol=0, atol=1e-12)


def check_attention_rows_subset(varlen_attention):
    rng = np.random.default_rng(24)
    cu = [0, 10, 45, 46]
    q, k, v = (rng.standard_normal((46, 2, 8)) for _ in range(3))
    o, lse = varlen_attention(q, k, v, cu)
    rows = np.array([0, 9, 10, 30, 45])
    o2, lse2 = varlen_attention(q, k, v, cu, rows=rows, chunk=2)
    assert np.array_equal(o2, o[rows]) or np.allclose(o2, o[rows], rtol=0, atol=1e-14)
    assert np.allclose(lse2, lse[:, rows], rtol=0, atol=1e-14)


# ----------------------------------------------------------------------- gate
def check_gate(gated_residual, adaln_params, pack_build):
    w = make_random_pack(40, S=2, H=2, D=8, rope_axes=2)
    p = pack_build(w.descs, 2)
    x = w.f32("x")
    o = np.random.default_rng(1).standard_normal((w.T, w.H, w.D))
    # a conditioning vector that is 1 in its first entry and a W whose gate
    # columns read that entry: gate = 1, so y = x + O
    c = np.zeros((w.S, 4))
    c[:, 0] = 1.0
    W = np.zeros((4, 6 * w.hid))
    for m in range(2):
        W[0, (3 * m + 2) * w.hid:(3 * m + 3) * w.hid] = 1.0
    mod = adaln_params(c, W, w.hid)
    y = gated_residual(x, o, mod, p["tok_sample"], p["tok_mod"])
    assert np.allclose(y, x + o.reshape(w.T, w.hid), rtol=0, atol=1e-15)
    # brute force with a random map
    mod = adaln_params(w.c, w.W, w.hid)
    y = gated_residual(x, o, mod, p["tok_sample"], p["tok_mod"])
    for t in range(w.T):
        s, m = int(p["tok_sample"][t]), int(p["tok_mod"][t])
        ref = brute.brute_gate_row(x[t].tolist(), o[t].reshape(-1).tolist(), mod[s, m, 2].tolist())
        assert np.allclose(y[t], ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Packed CFG combine  ([cfg])
# ---------------------------------------------------------------------------
_CFG_DESCS = [(1, 3, 4, 5), (0, 0, 0, 7), (1, 3, 4, 2), (1, 2, 2, 1), (1, 2, 2, 6)]
_CFG_PAIRS = [(0, 2), (4, 3)]  # (cond, uncond): 12 and 4 image tokens


def check_cfg_special_weights(cfg_combine):
    """w = 0 returns the unconditional branch, w = 1 the conditional one, and
    equal branches are left alone at any w (guidance has nothing to act on)."""
    rng = np.random.default_rng(50)
    T = sum(F * H * W + L for (F, H, W, L) in _CFG_DESCS)
    # dyadic values, as bf16 inputs are: u + (c - u) is then exactly c in float64
    v = rng.integers(-512, 512, size=(T, 8)) / 64.0
    cu = np.concatenate([[0], np.cumsum([F * H * W + L for (F, H, W, L) in _CFG_DESCS])])
    want_u = np.concatenate([v[cu[3]:cu[3] + 4] if u == 3 else v[cu[2]:cu[2] + 12]
                             for (_c, u) in _CFG_PAIRS])
    want_c = np.concatenate([v[cu[0]:cu[0] + 12], v[cu[4]:cu[4] + 4]])
    assert np.array_equal(cfg_combine(v, _CFG_DESCS, _CFG_PAIRS, 0.0), want_u)
    assert np.array_equal(cfg_combine(v, _CFG_DESCS, _CFG_PAIRS, 1.0), want_c)
    v2 = v.copy()
    v2[cu[2]:cu[2] + 12] = v2[cu[0]:cu[0] + 12]
    v2[cu[3]:cu[3] + 4] = v2[cu[4]:cu[4] + 4]
    for w in (0.0, 3.5, -2.0):
        assert np.array_equal(cfg_combine(v2, _CFG_DESCS, _CFG_PAIRS, w), want_c)


def check_cfg_row_map(cfg_combine):
    """Which rows are combined: with v[t] = t in every channel, row i of pair
    (c, u) is cu[u] + i + w * (cu[c] - cu[u]) (closed form of the row map:
    image tokens first, same index i in both samples), and text rows never
    enter."""
    T = sum(F * H * W + L for (F, H, W, L) in _CFG_DESCS)
    v = np.repeat(np.arange(T, dtype=np.float64)[:, None], 3, axis=1)
    cu = [0, 17, 24, 38, 43, 53]
    w = 4.25
    got = cfg_combine(v, _CFG_DESCS, _CFG_PAIRS, w)
    want = [cu[2] + i + w * (cu[0] - cu[2]) for i in range(12)] + \
           [cu[3] + i + w * (cu[4] - cu[3]) for i in range(4)]
    assert got.shape == (16, 3)
    assert np.allclose(got, np.repeat(np.array(want)[:, None], 3, axis=1), rtol=0, atol=1e-12)


def check_cfg_pack_order(cfg_combine):
    """Reordering the samples of the pack (and renumbering the pairs) leaves the
    guided output unchanged."""
    rng = np.random.default_rng(51)
    n = [F * H * W + L for (F, H, W, L) in _CFG_DESCS]
    cu = np.concatenate([[0], np.cumsum(n)])
    v = rng.standard_normal((cu[-1], 5))
    perm = [3, 0, 4, 2, 1]  # new position -> old sample
    descs2 = [_CFG_DESCS[o] for o in perm]
    v2 = np.concatenate([v[cu[o]:cu[o + 1]] for o in perm])
    where = {o: i for i, o in enumerate(perm)}
    pairs2 = [(where[c], where[u]) for (c, u) in _CFG_PAIRS]
    a = cfg_combine(v, _CFG_DESCS, _CFG_PAIRS, 2.5)
    b = cfg_combine(v2, descs2, pairs2, 2.5)
    assert np.array_equal(a, b)


# ---------------------------------------------------------------------------
# Modality-specific linear layer  ([norm])
# ---------------------------------------------------------------------------
def _linear_case(seed=60, K=8, N=6):
    w = make_random_pack(seed, S=4, H=1, D=8, rope_axes=2, max_grid=4, max_text=5)
    p = oracle_pack_ids(w)
    rng = np.random.default_rng(seed + 1)
    x = rng.standard_normal((w.T, K))
    W = rng.standard_normal((2, N, K))
    return w, p, x, W


def oracle_pack_ids(w):
    """Modality of every token of a pack, written out from the descriptors
    (image tokens first in each sample, then text), independent of the
    oracle's pack_build."""
    mods = []
    for d in w.descs:
        mods += [0] * (d.frames * d.grid_h * d.grid_w) + [1] * d.n_text
    return np.asarray(mods, dtype=np.uint8)


def check_linear_vs_brute(modality_linear):
    w, tm, x, W = _linear_case()
    out = modality_linear(x, W, tm)
    assert out.shape == (w.T, W.shape[1])
    assert (tm == 0).any() and (tm == 1).any()
    for t in range(w.T):
        ref = brute.brute_linear_row(x[t].tolist(), W[int(tm[t])].tolist())
        assert np.allclose(out[t], ref, rtol=0, atol=1e-12)


def check_linear_routing(modality_linear):
    """Zero text weights zero exactly the text rows (and vice versa); identity
    weights return the input."""
    w, tm, x, W = _linear_case(K=6, N=6)
    W0 = W.copy()
    W0[1] = 0.0
    out = modality_linear(x, W0, tm)
    assert np.all(out[tm == 1] == 0.0) and np.all(out[tm == 0] != 0.0)
    W1 = W.copy()
    W1[0] = 0.0
    out = modality_linear(x, W1, tm)
    assert np.all(out[tm == 0] == 0.0) and np.all(out[tm == 1] != 0.0)
    eye = np.stack([np.eye(6), np.eye(6)])
    assert np.array_equal(modality_linear(x, eye, tm), x)


def check_gelu(gelu_tanh):
    """GELU(0) = 0; GELU(x) - GELU(-x) = x for any x (x Phi(x) has that odd part,
    and so does the tanh form); GELU(x) -> x and -> 0 far out; and within 2e-3
    of the exact x Phi(x) (the tanh form's known small deviation)."""
    from scipy.special import erf
    x = np.linspace(-8.0, 8.0, 4001)
    g = gelu_tanh(x)
    assert gelu_tanh(np.array([0.0]))[0] == 0.0
    assert np.allclose(g - gelu_tanh(-x), x, rtol=0, atol=1e-12)
    assert abs(gelu_tanh(np.array([12.0]))[0] - 12.0) < 1e-12
    assert abs(gelu_tanh(np.array([-12.0]))[0]) < 1e-12
    exact = 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))
    dev = np.abs(g - exact).max()
    assert 1e-5 < dev < 2e-3, dev  # close to, but not, the exact form


def check_linear_gelu(modality_linear, gelu_tanh):
    """act='gelu' is GELU applied after the linear map, row by row."""
    w, tm, x, W = _linear_case(seed=61)
    assert np.allclose(modality_linear(x, W, tm, "gelu"), gelu_tanh(modality_linear(x, W, tm)),
                       rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# The whole MMDiT block  ([norm], [fuse])
# ---------------------------------------------------------------------------
def _mmdit_case(seed=70, H=2, D=8, F=24, descs=None):
    descs = descs or [SampleDesc(1, 2, 3, 2), SampleDesc(1, 3, 2, 3)]
    w = make_random_pack(seed, S=len(descs), H=H, D=D, rope_axes=2, descs=descs)
    rng = np.random.default_rng(seed + 1)
    hid = H * D
    ws = dict(Wq=rng.standard_normal((2, hid, hid)) / 4, Wk=rng.standard_normal((2, hid, hid)) / 4,
              Wv=rng.standard_normal((2, hid, hid)) / 4, Wo=rng.standard_normal((2, hid, hid)) / 4,
              Wup=rng.standard_normal((2, F, hid)) / 4, Wdown=rng.standard_normal((2, hid, F)) / 5)
    mods = dict(mod_attn=rng.standard_normal((w.S, 2, 3, hid)) * 0.3,
                mod_mlp=rng.standard_normal((w.S, 2, 3, hid)) * 0.3)
    return w, ws, mods


def _ident(a):
    return np.asarray(a, dtype=np.float64)


def check_mmdit_vs_brute(mmdit_block_fwd, pack_build):
    w, ws, mods = _mmdit_case()
    p = pack_build(w.descs, 2)
    x = w.f32("x")
    y = mmdit_block_fwd(x, **ws, **mods, pack=p, H=w.H, D=w.D, rope_axes=2, store=_ident)
    ref = brute.brute_mmdit_block(x.tolist(), *[ws[k].tolist() for k in
                                                ("Wq", "Wk", "Wv", "Wo", "Wup", "Wdown")],
                                  mods["mod_attn"].tolist(), mods["mod_mlp"].tolist(),
                                  w.descs, w.H, w.D, 2)
    assert np.allclose(y, np.asarray(ref), rtol=0, atol=1e-10)


def check_mmdit_zero_branches(mmdit_block_fwd, pack_build):
    """Zero output and down-projection weights leave the input unchanged, bit
    for bit, whatever the rest."""
    w, ws, mods = _mmdit_case(seed=71)
    p = pack_build(w.descs, 2)
    x = w.f32("x")
    ws = dict(ws, Wo=np.zeros_like(ws["Wo"]), Wdown=np.zeros_like(ws["Wdown"]))
    y = mmdit_block_fwd(x, **ws, **mods, pack=p, H=w.H, D=w.D, rope_axes=2)
    assert np.array_equal(y, x.astype(np.float64))


def check_mmdit_reduces_to_path(mmdit_block_fwd, block_fwd, adaln_modulate, pack_build):
    """With identity q/k/v/out projections and a silent MLP branch (zero down
    projection), the block is the packed joint-attention path with q = k = v =
    adaLN(x)."""
    w, ws, mods = _mmdit_case(seed=72)
    p = pack_build(w.descs, 2)
    x = w.f32("x")
    hid = w.H * w.D
    eye = np.stack([np.eye(hid), np.eye(hid)])
    ws = dict(ws, Wq=eye, Wk=eye, Wv=eye, Wo=eye, Wdown=np.zeros_like(ws["Wdown"]))
    y = mmdit_block_fwd(x, **ws, **mods, pack=p, H=w.H, D=w.D, rope_axes=2, store=_ident)
    x1 = adaln_modulate(x, mods["mod_attn"], p["tok_sample"], p["tok_mod"])
    qkv = x1.reshape(w.T, w.H, w.D)
    _, ref, _ = block_fwd(x, qkv, qkv, qkv, mods["mod_attn"], p, 2)
    assert np.allclose(y, ref, rtol=0, atol=1e-12)


def check_mmdit_branch_gates(mmdit_block_fwd, pack_build):
    """The MLP branch answers to its own gate: zero MLP gates give the result of
    a zero down projection; zero attention gates leave the MLP acting on x."""
    w, ws, mods = _mmdit_case(seed=73)
    p = pack_build(w.descs, 2)
    x = w.f32("x")
    m2 = mods["mod_mlp"].copy()
    m2[:, :, 2] = 0.0
    a = mmdit_block_fwd(x, **ws, mod_attn=mods["mod_attn"], mod_mlp=m2, pack=p, H=w.H, D=w.D,
                        rope_axes=2, store=_ident)
    b = mmdit_block_fwd(x, **dict(ws, Wdown=np.zeros_like(ws["Wdown"])), **mods, pack=p, H=w.H,
                        D=w.D, rope_axes=2, store=_ident)
    assert np.allclose(a, b, rtol=0, atol=1e-13)
    assert not np.allclose(a, x, atol=1e-6)


# ---------------------------------------------------------------------------
# Attention backward
# ---------------------------------------------------------------------------
def check_attention_bwd_vs_autograd(varlen_attention_bwd):
    """Per sample, torch autograd through fp64 SDPA (a library routine) gives
    the same gradients; samples of the pack never mix."""
    w = make_random_pack(80, S=3, H=2, D=16, rope_axes=2, max_grid=4, max_text=6)
    from oracle.mf_oracle import pack_build as _pb
    cu = _pb(w.descs, 2)["cu_seqlens"]
    rng = np.random.default_rng(81)
    q, k, v = w.f32("q"), w.f32("k"), w.f32("v")
    d_o = rng.standard_normal(q.shape)
    dq, dk, dv = varlen_attention_bwd(q, k, v, d_o, cu)
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        if hi == lo:
            continue
        t = [torch.tensor(a[lo:hi].transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
             for a in (q, k, v)]
        o = torch.nn.functional.scaled_dot_product_attention(*t)
        o.backward(torch.tensor(d_o[lo:hi].transpose(1, 0, 2), dtype=torch.float64))
        for got, ref in zip((dq, dk, dv), t):
            assert np.allclose(got[lo:hi], ref.grad.numpy().transpose(1, 0, 2), rtol=0, atol=1e-11)


def check_attention_bwd_finite_diff(varlen_attention_bwd, varlen_attention):
    """Directional derivatives of L = sum(dO * O) by central differences of the
    forward match <grad, direction> for q, k and v."""
    w = make_random_pack(82, S=2, H=2, D=8, rope_axes=2, max_grid=3, max_text=4)
    from oracle.mf_oracle import pack_build as _pb
    cu = _pb(w.descs, 2)["cu_seqlens"]
    rng = np.random.default_rng(83)
    q, k, v = (w.f32(n).astype(np.float64) for n in ("q", "k", "v"))
    d_o = rng.standard_normal(q.shape)
    grads = varlen_attention_bwd(q, k, v, d_o, cu)

    def loss(qq, kk, vv):
        return float((varlen_attention(qq, kk, vv, cu)[0] * d_o).sum())

    eps = 1e-6
    for i, g in enumerate(grads):
        u = rng.standard_normal(q.shape)
        args_p = [q, k, v]
        args_m = [q, k, v]
        args_p[i] = args_p[i] + eps * u
        args_m[i] = args_m[i] - eps * u
        fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert abs(fd - float((g * u).sum())) < 1e-6 * max(1.0, abs(fd)), (i, fd)


def _bwd_case(seed: int, rope_axes: int, D: int = 8, H: int = 2):
    """A small random pack with modulation vectors of order 0.3 (so that every
    term of the block matters) and upstream gradients."""
    w = make_random_pack(seed, S=3, H=H, D=D, rope_axes=rope_axes, max_grid=3, max_text=4)
    from oracle.mf_oracle import pack_build as _pb
    pack = _pb(w.descs, rope_axes)
    rng = np.random.default_rng(seed + 1)
    T, hid = w.T, H * D
    x = w.f32("x").astype(np.float64)
    q, k, v = (w.f32(n).astype(np.float64) for n in ("q", "k", "v"))
    mod = 0.3 * rng.standard_normal((w.S, 2, 3, hid))
    dy = rng.standard_normal((T, hid))
    dxm = rng.standard_normal((T, hid))
    return pack, x, q, k, v, mod, dy, dxm, rng


def check_block_bwd_finite_diff(block_bwd, block_fwd):
    """Directional derivatives of L = <dy, y> + <dx_mod, x_mod> by central
    differences of the forward match <grad, direction> for x, q, k, v and the
    modulation vectors (2D and 3D RoPE packs)."""
    for seed, axes, D in ((90, 2, 8), (92, 3, 16)):
        pack, x, q, k, v, mod, dy, dxm, rng = _bwd_case(seed, axes, D)
        grads = block_bwd(dy, dxm, x, q, k, v, mod, pack, axes)

        def loss(xx, qq, kk, vv, mm):
            xm, y, _ = block_fwd(xx, qq, kk, vv, mm, pack, axes)
            return float((y * dy).sum() + (xm * dxm).sum())

        base = [x, q, k, v, mod]
        eps = 1e-6
        for i, g in enumerate(grads):
            u = rng.standard_normal(base[i].shape)
            plus = list(base)
            minus = list(base)
            plus[i] = base[i] + eps * u
            minus[i] = base[i] - eps * u
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            got = float((g * u).sum())
            assert abs(fd - got) < 1e-5 * max(1.0, abs(fd)), (axes, i, fd, got)


def check_adaln_bwd_vs_torch_layer_norm(adaln_modulate_bwd):
    """torch autograd through its own layer_norm (a library routine) and the
    per-token gather of shift / scale gives the same dx and the same per-sample,
    per-modality sums of the shift and scale gradients."""
    pack, x, q, k, v, mod, dy, dxm, rng = _bwd_case(94, 2)
    S, hid = mod.shape[0], x.shape[1]
    eps = 1e-6
    dx, dmod = adaln_modulate_bwd(dxm, x, mod, pack["tok_sample"], pack["tok_mod"], S, eps)
    xt = torch.tensor(x, requires_grad=True)
    mt = torch.tensor(mod, requires_grad=True)
    ts = torch.tensor(pack["tok_sample"].astype(np.int64))
    tm = torch.tensor(pack["tok_mod"].astype(np.int64))
    xhat = torch.nn.functional.layer_norm(xt, (hid,), eps=eps)
    out = xhat * (1.0 + mt[ts, tm, 1]) + mt[ts, tm, 0]
    out.backward(torch.tensor(dxm))
    assert np.allclose(dx, xt.grad.numpy(), rtol=0, atol=1e-10)
    assert np.allclose(dmod, mt.grad.numpy(), rtol=0, atol=1e-10)


def check_adaln_bwd_invariants(adaln_modulate_bwd):
    """LayerNorm ignores a constant added to a row, so each row of dx sums to 0;
    with eps = 0 it also ignores a row's scale, so dx is orthogonal to the
    centred row."""
    pack, x, q, k, v, mod, dy, dxm, rng = _bwd_case(96, 2)
    S = mod.shape[0]
    dx, _ = adaln_modulate_bwd(dxm, x, mod, pack["tok_sample"], pack["tok_mod"], S, 1e-6)
    assert np.abs(dx.sum(axis=1)).max() < 1e-10
    dx0, _ = adaln_modulate_bwd(dxm, x, mod, pack["tok_sample"], pack["tok_mod"], S, 0.0)
    xc = x - x.mean(axis=1, keepdims=True)
    assert np.abs((dx0 * xc).sum(axis=1)).max() < 1e-9


def check_rope_bwd_adjoint(rope_bwd, rope_apply):
    """rope_bwd is the adjoint of rope_apply: <R x, y> = <x, R^T y> for random
    x, y, and R^T R x = x (2D packs and 3D packs with unrotated leftover
    channels)."""
    for seed, axes, D in ((98, 2, 8), (99, 3, 16)):
        pack, x, q, k, v, mod, dy, dxm, rng = _bwd_case(seed, axes, D)
        a = rng.standard_normal(q.shape)
        b = rng.standard_normal(q.shape)
        lhs = float((rope_apply(a, pack["pos_ids"], axes) * b).sum())
        rhs = float((a * rope_bwd(b, pack["pos_ids"], axes)).sum())
        assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(lhs))
        back = rope_bwd(rope_apply(a, pack["pos_ids"], axes), pack["pos_ids"], axes)
        assert np.abs(back - a).max() < 1e-12


def check_adaln_params_bwd_adjoint(adaln_params_bwd, adaln_params):
    """mod = c W is bilinear: <dmod, c' W> = <dc, c'> and <dmod, c W'> = <dW, W'>
    for any directions c', W'."""
    rng = np.random.default_rng(100)
    S, C, hid = 3, 5, 4
    c = rng.standard_normal((S, C))
    W = rng.standard_normal((C, 6 * hid))
    dmod = rng.standard_normal((S, 2, 3, hid))
    dc, dW = adaln_params_bwd(dmod, c, W)
    c2 = rng.standard_normal((S, C))
    W2 = rng.standard_normal((C, 6 * hid))
    assert abs(float((adaln_params(c2, W, hid) * dmod).sum()) - float((dc * c2).sum())) < 1e-10
    assert abs(float((adaln_params(c, W2, hid) * dmod).sum()) - float((dW * W2).sum())) < 1e-10


def check_gelu_bwd_vs_torch(gelu_tanh_bwd):
    """torch autograd through its own tanh-form GELU (a library routine) gives
    the same derivative, over a range that covers both tails."""
    z = np.linspace(-8.0, 8.0, 2001)
    dh = np.random.default_rng(101).standard_normal(z.shape)
    zt = torch.tensor(z, requires_grad=True)
    torch.nn.functional.gelu(zt, approximate="tanh").backward(torch.tensor(dh))
    assert np.allclose(gelu_tanh_bwd(z, dh), zt.grad.numpy(), rtol=0, atol=1e-12)


def check_linear_bwd_vs_autograd(modality_linear_bwd):
    """torch autograd (float64) through out[t] = x[t] @ W[m(t)]^T, the rows of
    each modality routed by index (a library matmul per modality), gives the
    same dx and dW; a modality without tokens gets dW[m] = 0."""
    rng = np.random.default_rng(103)
    T, K, N = 37, 24, 16
    x = rng.standard_normal((T, K))
    W = rng.standard_normal((2, N, K))
    dout = rng.standard_normal((T, N))
    for tok_mod in (rng.integers(0, 2, T).astype(np.uint8), np.zeros(T, dtype=np.uint8)):
        xt = torch.tensor(x, requires_grad=True)
        Wt = torch.tensor(W, requires_grad=True)
        out = torch.zeros((T, N), dtype=torch.float64)
        for m in (0, 1):
            idx = torch.tensor(np.nonzero(tok_mod == m)[0])
            out = out.index_add(0, idx, xt[idx] @ Wt[m].T)
        out.backward(torch.tensor(dout))
        dx, dW = modality_linear_bwd(x, W, tok_mod, dout)
        assert np.allclose(dx, xt.grad.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(dW, Wt.grad.numpy(), rtol=0, atol=1e-12)
    assert np.all(dW[1] == 0.0)  # the last case has no text token


def check_mmdit_bwd_finite_diff(mmdit_block_bwd, mmdit_block_fwd):
    """Directional derivatives of L = <dy, y> of the unrounded whole block by
    central differences match <grad, direction> for x, all six weight tensors
    and both modulation maps."""
    w = make_random_pack(102, S=2, H=2, D=8, rope_axes=2, max_grid=3, max_text=3)
    from oracle.mf_oracle import pack_build as _pb
    pack = _pb(w.descs, 2)
    rng = np.random.default_rng(103)
    T, hid = w.T, 16
    F = 4 * hid
    x = rng.standard_normal((T, hid))
    Ws = {n: rng.standard_normal((2, hid, hid)) / 4 for n in ("Wq", "Wk", "Wv", "Wo")}
    Ws["Wup"] = rng.standard_normal((2, F, hid)) / 4
    Ws["Wdown"] = rng.standard_normal((2, hid, F)) / 8
    mods = {n: 0.3 * rng.standard_normal((w.S, 2, 3, hid)) for n in ("mod_attn", "mod_mlp")}
    dy = rng.standard_normal((T, hid))
    args = dict(x=x, **Ws, **mods)
    order = ("x", "Wq", "Wk", "Wv", "Wo", "Wup", "Wdown", "mod_attn", "mod_mlp")

    def loss(a):
        y = mmdit_block_fwd(*[a[n] for n in order], pack, 2, 8, 2, store=lambda t: t)
        return float((y * dy).sum())

    grads = mmdit_block_bwd(dy, *[args[n] for n in order], pack, 2, 8, 2)
    eps = 1e-6
    for n in order:
        u = rng.standard_normal(args[n].shape)
        plus, minus = dict(args), dict(args)
        plus[n] = args[n] + eps * u
        minus[n] = args[n] - eps * u
        fd = (loss(plus) - loss(minus)) / (2 * eps)
        got = float((grads[n] * u).sum())
        assert abs(fd - got) < 1e-5 * max(1.0, abs(fd)), (n, fd, got)


def check_attention_bwd_vs_brute(varlen_attention_bwd):
    """The vectorised backward agrees with the scalar loops of
    oracle.brute.brute_attention_bwd (written independently: per query row, the
    mean of dp under p instead of rowsum(dO * O)) on tiny packs with an empty
    and a one-token sample."""
    from oracle.brute import brute_attention_bwd
    from packgen import SampleDesc
    descs = [SampleDesc(1, 2, 3, 2), SampleDesc(0, 0, 0, 0), SampleDesc(1, 1, 1, 0),
             SampleDesc(1, 2, 2, 1)]
    w = make_random_pack(104, S=len(descs), H=2, D=4, rope_axes=2, descs=descs)
    from oracle.mf_oracle import pack_build as _pb
    cu = [int(c) for c in _pb(w.descs, 2)["cu_seqlens"]]
    rng = np.random.default_rng(105)
    q, k, v = w.f32("q"), w.f32("k"), w.f32("v")
    d_o = rng.standard_normal(q.shape)
    got = varlen_attention_bwd(q, k, v, d_o, cu)
    ref = brute_attention_bwd(q.tolist(), k.tolist(), v.tolist(), d_o.tolist(), cu)
    for g, r in zip(got, ref):
        assert np.allclose(g, np.array(r), rtol=0, atol=1e-12)
