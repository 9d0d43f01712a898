"""Backward of the per-sample RoPE (mf_rope_bwd, through the C ABI) against the
float64 oracle's transposed rotation on the same seeded inputs: 2D and 3D packs
(3D with unrotated leftover channels), in place and out of place, and the edit
pack at full size on sampled rows. Same bf16 comparison rule as the forward
rotation (max-abs 2e-2, relative RMS 5e-3)."""

import numpy as np
import pytest
import torch

import oracle
from packgen import SampleDesc, draw_grad_bits, make_random_pack, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import resolution_packed_diffusion_b200 as mf  # noqa: E402
from gpu_util import (DevicePack, assert_bf16_close, dev_bf16, host_f32,  # noqa: E402
                      oracle_pack, sample_rows)
from packgen import bf16_bits_to_f32  # noqa: E402

PACKS = [
    # (descs, H, D, rope_axes)
    ([SampleDesc(1, 16, 16, 20), SampleDesc(1, 8, 32, 12)], 2, 64, 2),
    ([SampleDesc(1, 12, 20, 33), SampleDesc(0, 0, 0, 5)], 3, 128, 2),
    ([SampleDesc(2, 6, 5, 7), SampleDesc(1, 9, 4, 2)], 2, 128, 3),   # 42|42|42 + 2 kept
    ([SampleDesc(2, 8, 8, 9)], 2, 64, 3),                              # 20|20|20 + 4 kept
]


@pytest.mark.parametrize("k", range(len(PACKS)))
@pytest.mark.parametrize("in_place", [False, True], ids=["out", "inplace"])
def test_rope_bwd_small_packs(k, in_place):
    descs, H, D, axes = PACKS[k]
    w = make_random_pack(1200 + k, S=len(descs), H=H, D=D, rope_axes=axes, descs=descs)
    dp = DevicePack(w)
    pack = oracle_pack(w)
    gq_bits = draw_grad_bits(1300 + k, (w.T, H, D))
    gk_bits = draw_grad_bits(1400 + k, (w.T, H, D))
    gq, gk = dev_bf16(gq_bits), dev_bf16(gk_bits)
    if in_place:
        dq, dk = gq, gk
    else:
        dq, dk = torch.empty_like(gq), torch.empty_like(gk)
    mf.mf_rope_bwd(gq, gk, dp.pos, w.T, H, D, axes, w.base, dq, dk)
    assert mf.mf_get_error() == mf.MF_OK
    for name, got, bits in (("dq", dq, gq_bits), ("dk", dk, gk_bits)):
        ref = oracle.rope_bwd(bf16_bits_to_f32(bits), pack["pos_ids"], axes, w.base)
        assert_bf16_close(host_f32(got), ref, "RoPE backward " + name)


def test_rope_bwd_undoes_the_rotation():
    """mf_rope_bwd(mf_rope_apply(q)) returns q up to two bf16 roundings."""
    descs, H, D, axes = PACKS[2]
    w = make_random_pack(1250, S=len(descs), H=H, D=D, rope_axes=axes, descs=descs)
    dp = DevicePack(w)
    rot = torch.empty_like(dp.q)
    back = torch.empty_like(dp.q)
    mf.mf_rope_apply(dp.q, None, dp.pos, w.T, H, D, axes, w.base, rot, None)
    mf.mf_rope_bwd(rot, None, dp.pos, w.T, H, D, axes, w.base, back, None)
    assert mf.mf_get_error() == mf.MF_OK
    assert_bf16_close(host_f32(back), w.f32("q").astype(np.float64), "R^T R q")


def test_rope_bwd_edit_pack_sampled_rows():
    w = make_workload(4)
    dp = DevicePack(w)
    pack = oracle_pack(w)
    g_bits = draw_grad_bits(4, (w.T, w.H, w.D))
    g = dev_bf16(g_bits)
    out = torch.empty_like(g)
    mf.mf_rope_bwd(g, None, dp.pos, w.T, w.H, w.D, w.rope_axes, w.base, out, None)
    assert mf.mf_get_error() == mf.MF_OK
    rows = sample_rows(pack["cu_seqlens"], 64, 4)
    ref = oracle.rope_bwd(bf16_bits_to_f32(g_bits)[rows], pack["pos_ids"][rows], w.rope_axes,
                          w.base)
    assert_bf16_close(host_f32(out)[rows], ref, "RoPE backward, edit pack")
