"""Backward of the packed joint attention (mf_varlen_attn_bwd, through the C
ABI) against the float64 oracle on the same seeded inputs.

The GPU side runs the library's own forward for O and the log-sum-exp, then
the backward; the oracle differentiates the same bf16 q, k, v and dO in float64
(its own forward inside). Small packs are compared in full (ragged tiles, empty
samples, both head sizes, several query and key tiles per sample); the
training, packed-CFG, edit and large packs at full size on two heads (the oracle
works head by head, so a head subset is the same computation).

Tolerance: the stated one for bf16-in / fp32-accumulate outputs, relative RMS
error <= 5e-3, taken per tensor and per sample (the gradients' scale varies
from sample to sample), and a largest error <= 2^-5 of the largest reference
magnitude of that tensor and sample in place of the absolute 2e-2 (|dq| is of
the order of 1e-2 at these shapes, so an absolute bound would not test it).
Sources of error: P and dS are rounded to bf16 before their products (relative
error up to 2^-9 each), O enters rowsum(dO * O) as bf16, and each output is
stored as bf16; every output element is a sum of many such terms with
independent rounding.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from packgen import SampleDesc, draw_grad_bits, make_random_pack, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import resolution_packed_diffusion_b200 as mf  # noqa: E402
from gpu_util import (DevicePack, assert_grad_close, dev_bf16, host_f32, oracle_pack,  # noqa: E402
                      zero_grad_bound)


def gpu_backward(dp: DevicePack, d_o: torch.Tensor, heads=None):
    """Forward (for O and LSE) then backward on the device. ``heads`` selects a
    head subset by slicing the inputs (contiguous copies)."""
    q, k, v = dp.q, dp.k, dp.v
    H = dp.H
    if heads is not None:
        q, k, v = (t[:, heads].contiguous() for t in (q, k, v))
        d_o = d_o[:, heads].contiguous()
        H = len(heads)
    T, D = dp.T, dp.D
    scale = 1.0 / math.sqrt(D)
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda")
    mf.mf_varlen_attn_fwd(q, k, v, dp.cu_d, dp.cu_h, dp.S, H, D, scale, None, 2, 10000.0, o, lse,
                          None, 0)
    dq, dk, dv = (torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    ws_bytes = mf.mf_attn_bwd_workspace_size(T, dp.S, H, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    mf.mf_varlen_attn_bwd(q, k, v, o, d_o, lse, dp.cu_d, dp.cu_h, dp.S, H, D, scale, dq, dk, dv,
                          ws, ws_bytes)
    assert mf.mf_get_error() == mf.MF_OK
    return host_f32(dq), host_f32(dk), host_f32(dv)


def check(w, heads=None, seed=0):
    dp = DevicePack(w)
    pack = oracle_pack(w)
    cu = pack["cu_seqlens"]
    g_bits = draw_grad_bits(seed, (w.T, w.H, w.D))
    d_o = dev_bf16(g_bits)
    dq, dk, dv = gpu_backward(dp, d_o, heads)
    sel = slice(None) if heads is None else heads
    f = lambda name: w.f32(name)[:, sel]  # noqa: E731
    from packgen import bf16_bits_to_f32
    ref = oracle.varlen_attention_bwd(f("q"), f("k"), f("v"), bf16_bits_to_f32(g_bits)[:, sel], cu)
    ztol = zero_grad_bound(f("q"), f("k"), f("v"), bf16_bits_to_f32(g_bits)[:, sel], w.D)
    stats = []
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        stats += assert_grad_close(g, r, cu, name, ztol if name != "dv" else 0.0)
    for st in stats:
        print("%s sample %d (%d tokens): rel-rms %.3g, max/max|ref| %.3g" % st)
    return stats


SMALL_PACKS = [
    # (descs, H, D)
    ([SampleDesc(1, 16, 16, 20), SampleDesc(1, 8, 32, 12)], 2, 64),          # 276 + 268 tokens
    ([SampleDesc(1, 4, 4, 0), SampleDesc(0, 0, 0, 0), SampleDesc(1, 3, 3, 5)], 2, 128),  # empty
    ([SampleDesc(1, 16, 16, 255)], 1, 128),                                   # 511: ragged tiles
    ([SampleDesc(1, 20, 20, 113), SampleDesc(1, 1, 1, 0), SampleDesc(1, 16, 24, 7)], 3, 128),
    ([SampleDesc(1, 16, 16, 0), SampleDesc(1, 16, 16, 1)], 4, 64),            # 256 and 257
]


@pytest.mark.parametrize("k", range(len(SMALL_PACKS)))
def test_backward_small_packs_full_compare(k):
    descs, H, D = SMALL_PACKS[k]
    w = make_random_pack(900 + k, S=len(descs), H=H, D=D, rope_axes=2, descs=descs)
    check(w, seed=900 + k)


@pytest.mark.parametrize("idx", [2, 3, 4, 5],
                         ids=["training_pack", "cfg_pack", "edit_pack", "large_pack"])
def test_backward_full_size_two_heads(idx):
    """The workloads at full size; heads 0 and H-1 are compared (the oracle's
    cost grows with n^2 per head). The large pack's 16896-token sample is the
    longest key walk of the kernel and the most dQ reductions per query tile;
    the oracle holds its n x n score, probability and gradient matrices in
    float64 (about 2.3 GB each)."""
    need_gb = {2: 4, 3: 4, 4: 12, 5: 16}[idx]
    try:
        import psutil
        free_gb = psutil.virtual_memory().available / 2 ** 30
    except ImportError:
        free_gb = float("inf")
    if free_gb < 2 * need_gb:
        pytest.skip(f"the float64 oracle needs about {need_gb} GB of host memory "
                    f"({free_gb:.0f} GB available)")
    w = make_workload(idx)
    check(w, heads=[0, w.H - 1], seed=idx)


def test_backward_all_heads_match_head_subset():
    """The launch over all heads computes, for heads 0 and H-1, what a launch
    over those two heads alone computes (work items of other heads do not
    disturb them): dK and dV bit for bit; dQ sums key tiles in whatever order
    their reductions land, so it differs by fp32 reordering of partial sums
    that can cancel (bf16 rounding then moves it by an ulp of the result or
    so): bounded by 2^-8 of the largest |dQ| of the head, far below any effect
    of a disturbed item (of the order of the values themselves)."""
    w = make_workload(3)
    dp = DevicePack(w)
    d_o = dev_bf16(draw_grad_bits(3, (w.T, w.H, w.D)))
    full = gpu_backward(dp, d_o)
    sub = gpu_backward(dp, d_o, heads=[0, w.H - 1])
    np.testing.assert_array_equal(full[1][:, [0, w.H - 1]], sub[1])
    np.testing.assert_array_equal(full[2][:, [0, w.H - 1]], sub[2])
    a, b = full[0][:, [0, w.H - 1]].astype(np.float64), sub[0].astype(np.float64)
    bound = 2.0 ** -8 * np.abs(b).max(axis=(0, 2), keepdims=True)
    assert (np.abs(a - b) <= bound).all()


def test_backward_rejects_aliasing_and_short_workspace():
    w = make_random_pack(950, S=2, H=2, D=64, rope_axes=2,
                         descs=[SampleDesc(1, 8, 8, 3), SampleDesc(1, 4, 4, 2)])
    dp = DevicePack(w)
    T, H, D = dp.T, dp.H, dp.D
    o = torch.zeros((T, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((H, T), dtype=torch.float32, device="cuda")
    dq, dk, dv = (torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    ws_bytes = mf.mf_attn_bwd_workspace_size(T, dp.S, H, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    with pytest.raises(mf.MFError):  # dq aliases q
        mf.mf_varlen_attn_bwd(dp.q, dp.k, dp.v, o, o, lse, dp.cu_d, dp.cu_h, dp.S, H, D, 0.125,
                              dp.q, dk, dv, ws, ws_bytes)
    with pytest.raises(mf.MFError):  # workspace too small
        mf.mf_varlen_attn_bwd(dp.q, dp.k, dp.v, o, o, lse, dp.cu_d, dp.cu_h, dp.S, H, D, 0.125,
                              dq, dk, dv, ws, ws_bytes - 256)
    with pytest.raises(mf.MFError):  # dk and dv the same buffer
        mf.mf_varlen_attn_bwd(dp.q, dp.k, dp.v, o, o, lse, dp.cu_d, dp.cu_h, dp.S, H, D, 0.125,
                              dq, dk, dk, ws, ws_bytes)
    assert mf.mf_get_error() == mf.MF_OK
