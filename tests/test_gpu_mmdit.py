"""One NR-MMDiT block forward (adaLN, per-modality projections on tcgen05, RoPE,
packed joint attention, gated residuals, GELU MLP) on the GPU through the C
ABI, against the oracle's block with the same bf16 storage of intermediates."""

import math

import numpy as np
import pytest
import torch

import oracle
import resolution_packed_diffusion_b200 as mf
from gpu_util import assert_block_close, dev_bf16, host_f32, sample_rows
from packgen import SampleDesc, f32_to_bf16_bits, make_random_pack, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _weights(rng, hid, F):
    def w(n, k):
        return f32_to_bf16_bits((rng.standard_normal((2, n, k), dtype=np.float32)
                                 / np.float32(math.sqrt(k))).astype(np.float32))
    return dict(Wq=w(hid, hid), Wk=w(hid, hid), Wv=w(hid, hid), Wo=w(hid, hid), Wup=w(F, hid),
                Wdown=w(hid, F))


def _run(w, F, seed, rows=None):
    rng = np.random.default_rng(seed)
    hid = w.hid
    wb = _weights(rng, hid, F)
    mods = {k: (rng.standard_normal((w.S, 2, 3, hid), dtype=np.float32) * np.float32(0.3))
            for k in ("mod_attn", "mod_mlp")}
    cu_h, T = mf.mf_pack_build(w.descs, w.rope_axes, 0)
    cu_d = torch.empty(w.S + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 3), dtype=torch.int32, device="cuda")
    ts = torch.empty(T, dtype=torch.int32, device="cuda")
    tm = torch.empty(T, dtype=torch.uint8, device="cuda")
    mf.mf_pack_build(w.descs, w.rope_axes, 0, cu_d, pos, ts, tm)
    x = dev_bf16(w.x_bits.reshape(T, hid))
    dw = {k: dev_bf16(v) for k, v in wb.items()}
    dm = {k: torch.from_numpy(v).cuda() for k, v in mods.items()}
    y = torch.empty((T, hid), dtype=torch.bfloat16, device="cuda")
    ws_bytes = mf.mf_mmdit_workspace_size(T, w.H, w.D, F)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    mf.mf_mmdit_block_fwd(x, dw["Wq"], dw["Wk"], dw["Wv"], dw["Wo"], dw["Wup"], dw["Wdown"],
                          dm["mod_attn"], dm["mod_mlp"], w.descs, cu_d, cu_h, pos, ts, tm, w.S,
                          w.H, w.D, F, w.rope_axes, w.base, w.eps, y, ws, ws_bytes)
    assert mf.mf_get_error() == mf.MF_OK
    pack = oracle.pack_build(w.descs, w.rope_axes)
    from packgen import bf16_bits_to_f32
    ref = oracle.mmdit_block_fwd(
        w.f32("x").reshape(T, hid), *[bf16_bits_to_f32(wb[k]) for k in
                                      ("Wq", "Wk", "Wv", "Wo", "Wup", "Wdown")],
        mods["mod_attn"].astype(np.float64), mods["mod_mlp"].astype(np.float64), pack, w.H, w.D,
        w.rope_axes, w.base, w.eps, rows=rows)
    got = host_f32(y)
    return got if rows is None else got[rows], ref


@pytest.mark.parametrize("linear_pair", [0, 1], ids=["one_cta", "linear_cta_pairs"])
def test_mmdit_block_small_pack_every_row(linear_pair):
    descs = [SampleDesc(1, 9, 14, 5), SampleDesc(0, 0, 0, 33), SampleDesc(1, 11, 13, 2)]
    w = make_random_pack(970, S=3, H=2, D=128, rope_axes=2, descs=descs)
    mf.mf_set_linear_cta_pair(linear_pair)
    try:
        got, ref = _run(w, 512, 971)
    finally:
        mf.mf_set_linear_cta_pair(1)  # the library's default
    assert np.isfinite(got).all()
    assert_block_close(got, ref, "block y")


def test_mmdit_block_edit_pack_3d_rope():
    descs = [SampleDesc(2, 6, 7, 9), SampleDesc(2, 5, 5, 3)]
    w = make_random_pack(972, S=2, H=4, D=64, rope_axes=3, descs=descs)
    got, ref = _run(w, 256, 973)
    assert_block_close(got, ref, "block y (3D RoPE)")


def test_mmdit_block_cfg_pack_sampled_rows():
    """Full size: the packed-CFG workload, 24 heads x 128, MLP width 4 x 3072."""
    w = make_workload(3)
    pack = oracle.pack_build(w.descs, w.rope_axes)
    rows = sample_rows(pack["cu_seqlens"], 24, 974)
    got, ref = _run(w, 4 * w.hid, 975, rows=rows)
    assert np.isfinite(got).all()
    assert_block_close(got, ref, "block y rows")
