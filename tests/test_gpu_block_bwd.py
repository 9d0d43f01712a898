"""The backward of the whole path block, chained through the C ABI as a training
step runs it, against the float64 oracle's ``block_bwd`` on the same seeded
inputs and upstream gradients (dy of y, dx_mod of x_mod):

    forward state:  RoPE (mf_rope_apply), attention with LSE (mf_varlen_attn_fwd)
    gate:           mf_gated_residual_bwd   -> dO, dgate
    attention:      mf_varlen_attn_bwd      -> dq_r, dk_r, dv
    RoPE:           mf_rope_bwd             -> dq, dk
    adaLN:          mf_adaln_modulate_bwd   -> dx = dy + LayerNorm path, dshift, dscale

Every step consumes what the GPU produced before it (dO from the gate backward
feeds the attention backward, the rotated gradients feed the RoPE backward), so
a fault in how the steps fit together shows here even where each step passes on
its own. The 544-token pack is compared in full; the training pack at full size
on two heads for the attention-side outputs (every step but the LayerNorm is
separable by head column) and on every row for dx and the modulation sums.

Tolerances: dx (bf16) the block's rule, max-abs 2e-2 and relative RMS 5e-3;
dq, dk, dv the attention backward's rule (relative RMS 5e-3 per tensor and
sample, largest error 2^-5 of the largest reference magnitude); the fp32
modulation sums: dshift and dscale sum exact bf16 inputs, so they keep the fp32
summation bound of the gate / adaLN backward tests (3e-5 of the sum of |terms|);
dgate sums dy * O with O the GPU forward's bf16 output, whose own error is
bounded by the forward's max-abs rule, so |error| <= 2e-2 * sum|dy| and a
relative RMS error <= 5e-3 over each (sample, modality) row of sums.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from packgen import bf16_bits_to_f32, draw_grad_bits, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import resolution_packed_diffusion_b200 as mf  # noqa: E402
from gpu_util import (DevicePack, assert_bf16_close, assert_grad_close, dev_bf16,  # noqa: E402
                      host_f32, oracle_pack, sample_rows, zero_grad_bound)

SUM_REL = 3e-5


def gpu_block_bwd(dp: DevicePack, dy_bits, dxm_bits):
    """The chain on the device; returns host float arrays (dx, dq, dk, dv, dmod)."""
    w = dp.w
    T, S, H, D, hid = dp.T, dp.S, dp.H, dp.D, dp.hid
    dy, dxm = dev_bf16(dy_bits.reshape(T, hid)), dev_bf16(dxm_bits.reshape(T, hid))
    scale = 1.0 / math.sqrt(D)
    q_r, k_r = torch.empty_like(dp.q), torch.empty_like(dp.k)
    mf.mf_rope_apply(dp.q, dp.k, dp.pos, T, H, D, w.rope_axes, w.base, q_r, k_r)
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda")
    mf.mf_varlen_attn_fwd(q_r, k_r, dp.v, dp.cu_d, dp.cu_h, S, H, D, scale, None, w.rope_axes,
                          w.base, o, lse, None, 0)
    d_o = torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
    dmod = torch.full((S, 2, 3, hid), 7.0, dtype=torch.float32, device="cuda")
    mf.mf_gated_residual_bwd(dy, o, dp.mod, dp.tok_sample, dp.tok_mod, T, S, hid, d_o, dmod)
    dq_r, dk_r, dv = (torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
                      for _ in range(3))
    abw = mf.mf_attn_bwd_workspace_size(T, S, H, D)
    aws = torch.empty(abw, dtype=torch.uint8, device="cuda")
    mf.mf_varlen_attn_bwd(q_r, k_r, dp.v, o, d_o, lse, dp.cu_d, dp.cu_h, S, H, D, scale, dq_r,
                          dk_r, dv, aws, abw)
    dq, dk = torch.empty_like(dq_r), torch.empty_like(dk_r)
    mf.mf_rope_bwd(dq_r, dk_r, dp.pos, T, H, D, w.rope_axes, w.base, dq, dk)
    dx = torch.empty_like(dy)
    lbw = mf.mf_adaln_bwd_workspace_size(T)
    lws = torch.empty(max(lbw, 16), dtype=torch.uint8, device="cuda")
    mf.mf_adaln_modulate_bwd(dxm, dp.x, dp.mod, dp.tok_sample, dp.tok_mod, dy, T, S, hid, w.eps,
                             dx, dmod, lws, lbw)
    assert mf.mf_get_error() == mf.MF_OK
    return (host_f32(dx), host_f32(dq), host_f32(dk), host_f32(dv),
            dmod.cpu().numpy().astype(np.float64), host_f32(o).reshape(T, hid))


def seg_abs_sums(vals, ts, tm, S):
    out = np.zeros((S, 2, vals.shape[1]))
    np.add.at(out, (ts.astype(np.int64), tm.astype(np.int64)), np.abs(vals))
    return out


def check_sums(got, ref, mag, name):
    err = np.abs(got - ref)
    tol = SUM_REL * mag + 1e-6
    worst = int(np.argmax(err - tol))
    assert (err <= tol).all(), (f"{name}: |err| {err.flat[worst]:.3g} > {tol.flat[worst]:.3g} "
                                f"at {np.unravel_index(worst, err.shape)}")


def check_dgate(got, ref, dy, ts, tm, S, name="dgate"):
    err = np.abs(got - ref)
    tol = 2e-2 * seg_abs_sums(dy, ts, tm, S) + 1e-6
    assert (err <= tol).all(), f"{name}: max |err| - tol {float((err - tol).max()):.3g} > 0"
    # relative RMS over each (sample, modality) row of sums that has tokens
    for s in range(S):
        for m in range(2):
            r = ref[s, m]
            if not np.any(r):
                continue
            rr = float(np.linalg.norm(got[s, m] - r) / np.linalg.norm(r))
            assert rr <= 5e-3, f"{name}[{s}, {m}]: relative RMS {rr:.3g} > 5e-3"


def test_block_backward_chain_tiny_pack_full():
    w = make_workload(1)
    dp = DevicePack(w)
    pack = oracle_pack(w)
    T, S, H, D, hid = w.T, w.S, w.H, w.D, w.hid
    dy_bits = draw_grad_bits(2101, (T, hid))
    dxm_bits = draw_grad_bits(2102, (T, hid))
    dx, dq, dk, dv, dmod, _ = gpu_block_bwd(dp, dy_bits, dxm_bits)
    mod = oracle.adaln_params(w.c, w.W, hid)
    fdy, fdxm = bf16_bits_to_f32(dy_bits), bf16_bits_to_f32(dxm_bits)
    r_dx, r_dq, r_dk, r_dv, r_dmod = oracle.block_bwd(
        fdy, fdxm, w.f32("x"), w.f32("q"), w.f32("k"), w.f32("v"), mod, pack, w.rope_axes,
        w.base, w.eps)
    assert_bf16_close(dx, r_dx, "chain dx")
    cu = pack["cu_seqlens"]
    ztol = zero_grad_bound(w.f32("q"), w.f32("k"), w.f32("v"), fdy.reshape(T, H, D), D)
    assert_grad_close(dq, r_dq, cu, "chain dq", ztol)
    assert_grad_close(dk, r_dk, cu, "chain dk", ztol)
    assert_grad_close(dv, r_dv, cu, "chain dv")
    ts, tm = pack["tok_sample"], pack["tok_mod"]
    xhat = oracle.layer_norm_rows(w.f32("x"), w.eps)
    check_sums(dmod[:, :, 0], r_dmod[:, :, 0], seg_abs_sums(fdxm, ts, tm, S), "chain dshift")
    check_sums(dmod[:, :, 1], r_dmod[:, :, 1], seg_abs_sums(fdxm * xhat, ts, tm, S),
               "chain dscale")
    check_dgate(dmod[:, :, 2], r_dmod[:, :, 2], fdy, ts, tm, S, "chain dgate")


def test_block_backward_chain_training_pack():
    """Full size. The oracle's block_bwd runs on the columns of heads 0 and H-1
    with dx_mod = 0 (the gate, attention and RoPE steps act on each head's
    columns alone, and a zero dx_mod makes the LayerNorm path vanish), and its
    adaLN backward on every column for dx and the shift / scale sums."""
    w = make_workload(2)
    dp = DevicePack(w)
    pack = oracle_pack(w)
    T, S, H, D, hid = w.T, w.S, w.H, w.D, w.hid
    dy_bits = draw_grad_bits(2201, (T, hid))
    dxm_bits = draw_grad_bits(2202, (T, hid))
    dx, dq, dk, dv, dmod, _ = gpu_block_bwd(dp, dy_bits, dxm_bits)
    mod = oracle.adaln_params(w.c, w.W, hid)
    fdy, fdxm = bf16_bits_to_f32(dy_bits), bf16_bits_to_f32(dxm_bits)
    ts, tm = pack["tok_sample"], pack["tok_mod"]
    fx = w.f32("x")

    # LayerNorm path: every column, dx compared on sampled rows
    r_dxln, r_dmodln = oracle.adaln_modulate_bwd(fdxm, fx, mod, ts, tm, S, w.eps)
    rows = sample_rows(pack["cu_seqlens"], 64, 2203)
    assert_bf16_close(dx[rows], (fdy + r_dxln)[rows], "chain dx (sampled rows)")
    xhat = oracle.layer_norm_rows(fx, w.eps)
    check_sums(dmod[:, :, 0], r_dmodln[:, :, 0], seg_abs_sums(fdxm, ts, tm, S), "chain dshift")
    check_sums(dmod[:, :, 1], r_dmodln[:, :, 1], seg_abs_sums(fdxm * xhat, ts, tm, S),
               "chain dscale")

    # gate, attention and RoPE: the columns of two heads
    heads = [0, H - 1]
    cols = np.concatenate([np.arange(h * D, (h + 1) * D) for h in heads])
    sub = lambda a: np.ascontiguousarray(a[:, heads])  # noqa: E731
    _, r_dq, r_dk, r_dv, r_dmod = oracle.block_bwd(
        fdy[:, cols], np.zeros((T, len(cols))), fx[:, cols], sub(w.f32("q")), sub(w.f32("k")),
        sub(w.f32("v")), mod[..., cols], pack, w.rope_axes, w.base, w.eps)
    cu = pack["cu_seqlens"]
    ztol = zero_grad_bound(sub(w.f32("q")), sub(w.f32("k")), sub(w.f32("v")),
                           fdy[:, cols].reshape(T, len(heads), D), D)
    assert_grad_close(dq[:, heads], r_dq, cu, "chain dq", ztol)
    assert_grad_close(dk[:, heads], r_dk, cu, "chain dk", ztol)
    assert_grad_close(dv[:, heads], r_dv, cu, "chain dv")
    check_dgate(dmod[:, :, 2][..., cols], r_dmod[:, :, 2], fdy[:, cols], ts, tm, S,
                "chain dgate")
