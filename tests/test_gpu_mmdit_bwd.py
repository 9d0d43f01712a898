"""Backward of one NR-MMDiT block on the GPU (mf_mmdit_block_bwd: the forward
recomputed, then gates, linear layers on tcgen05 with transposed weights and
token-gathering transposes for the weight gradients, GELU, adaLN, attention and
RoPE backward) against the oracle's float64 ``mmdit_block_bwd``, every element
of every gradient, on both linear kernels.

Tolerance. The GPU chain stores ~25 intermediates in bf16 (the forward's x1, q,
k, v, their rotations, o, a, y1, x2, z, h, mlp; the backward's d_mlp, dz, dx2,
dy1, da, d_o, dq, dk, dv, dx1 and the gathered transposes), each a relative
rounding of at most 2^-9 (RMS 2^-9 / sqrt(3) = 1.1e-3); along the longest path
to a gradient about 16 of them compound, sqrt(16) * 1.1e-3 = 4.5e-3, on top of
the attention backward's own 5e-3 bound and the output's rounding. The bound is
therefore relative RMS 1e-2 per tensor (per sample for dx) and a maximum error of
2^-5 of the tensor's largest magnitude (as for the attention gradients); the
float64 oracle rounds nothing. Measured on a B200: dx 2.5e-3, dWq / dWk 6.7e-3 to
7.7e-3 (they pass through the attention and RoPE backward), the other weight and
modulation gradients 2.9e-3 to 4.9e-3; maxima at most 1.03e-2 of max|ref|."""

import math

import numpy as np
import pytest
import torch

import oracle
import resolution_packed_diffusion_b200 as mf
from gpu_util import dev_bf16, host_f32
from packgen import SampleDesc, bf16_bits_to_f32, f32_to_bf16_bits, make_random_pack

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

REL_RMS = 1e-2
MAX_REL = 2.0 ** -5


@pytest.fixture(params=[1, 0], ids=["linear_cta_pairs", "linear_one_cta"], autouse=True)
def linear_pair(request):
    mf.mf_set_linear_cta_pair(request.param)
    yield request.param
    mf.mf_set_linear_cta_pair(1)  # the library's default


def _close(got, ref, name):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape and np.isfinite(got).all(), name
    scale = np.abs(ref).max()
    if scale == 0.0:
        assert np.abs(got).max() == 0.0, f"{name}: expected exact zeros"
        return 0.0, 0.0
    rr = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    mr = float(np.abs(got - ref).max() / scale)
    print(f"{name}: rel RMS {rr:.2e}, max {mr:.2e} of max|ref|")
    assert rr <= REL_RMS, f"{name}: relative RMS {rr:.3g} > {REL_RMS}"
    assert mr <= MAX_REL, f"{name}: max error {mr:.3g} of max|ref| > {MAX_REL}"
    return rr, mr


def _run(w, F, seed):
    rng = np.random.default_rng(seed)
    hid, T, S = w.hid, w.T, w.S

    def wbits(n, k):
        return f32_to_bf16_bits((rng.standard_normal((2, n, k), dtype=np.float32)
                                 / np.float32(math.sqrt(k))).astype(np.float32))
    wb = dict(Wq=wbits(hid, hid), Wk=wbits(hid, hid), Wv=wbits(hid, hid), Wo=wbits(hid, hid),
              Wup=wbits(F, hid), Wdown=wbits(hid, F))
    mods = {k: (rng.standard_normal((S, 2, 3, hid), dtype=np.float32) * np.float32(0.3))
            for k in ("mod_attn", "mod_mlp")}
    dy_bits = f32_to_bf16_bits(rng.standard_normal((T, hid), dtype=np.float32))
    cu_h, T2 = mf.mf_pack_build(w.descs, w.rope_axes, 0)
    assert T2 == T
    cu_d = torch.empty(S + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, 3), dtype=torch.int32, device="cuda")
    ts = torch.empty(T, dtype=torch.int32, device="cuda")
    tm = torch.empty(T, dtype=torch.uint8, device="cuda")
    mf.mf_pack_build(w.descs, w.rope_axes, 0, cu_d, pos, ts, tm)
    x = dev_bf16(w.x_bits.reshape(T, hid))
    dy = dev_bf16(dy_bits)
    dw = {k: dev_bf16(v) for k, v in wb.items()}
    dm = {k: torch.from_numpy(v).cuda() for k, v in mods.items()}
    out = {n: torch.full(dw["W" + n[2:]].shape, float("nan"), dtype=torch.bfloat16, device="cuda")
           for n in ("dWq", "dWk", "dWv", "dWo", "dWup", "dWdown")}
    dx = torch.full((T, hid), float("nan"), dtype=torch.bfloat16, device="cuda")
    dmod = {k: torch.full((S, 2, 3, hid), float("nan"), device="cuda")
            for k in ("mod_attn", "mod_mlp")}
    ws_bytes = mf.mf_mmdit_bwd_workspace_size(T, S, w.H, w.D, F)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    mf.mf_mmdit_block_bwd(dy, x, dw["Wq"], dw["Wk"], dw["Wv"], dw["Wo"], dw["Wup"], dw["Wdown"],
                          dm["mod_attn"], dm["mod_mlp"], w.descs, cu_d, cu_h, pos, ts, tm, S, w.H,
                          w.D, F, w.rope_axes, w.base, w.eps, dx, out["dWq"], out["dWk"],
                          out["dWv"], out["dWo"], out["dWup"], out["dWdown"], dmod["mod_attn"],
                          dmod["mod_mlp"], ws, ws_bytes)
    assert mf.mf_get_error() == mf.MF_OK
    pack = oracle.pack_build(w.descs, w.rope_axes)
    ref = oracle.mmdit_block_bwd(
        bf16_bits_to_f32(dy_bits), w.f32("x").reshape(T, hid),
        *[bf16_bits_to_f32(wb[k]) for k in ("Wq", "Wk", "Wv", "Wo", "Wup", "Wdown")],
        mods["mod_attn"].astype(np.float64), mods["mod_mlp"].astype(np.float64), pack, w.H, w.D,
        w.rope_axes, w.base, w.eps)
    got = {"x": host_f32(dx), "mod_attn": dmod["mod_attn"].cpu().numpy(),
           "mod_mlp": dmod["mod_mlp"].cpu().numpy()}
    for n, t in out.items():
        got[n[1:]] = host_f32(t)
    return got, ref, pack


def _check_all(got, ref, pack, label):
    cu = pack["cu_seqlens"]
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        if hi > lo:
            _close(got["x"][lo:hi], ref["x"][lo:hi], f"{label} dx sample {s}")
    for n in ("Wq", "Wk", "Wv", "Wo", "Wup", "Wdown"):
        for m in (0, 1):
            _close(got[n][m], ref[n][m], f"{label} d{n}[{m}]")
    for n in ("mod_attn", "mod_mlp"):
        _close(got[n], ref[n], f"{label} d{n}")


def test_mmdit_block_bwd_small_pack():
    """Three samples (one text-only), 128-row tiles and 256-row blocks that mix
    modalities, hid 256, MLP width 512."""
    descs = [SampleDesc(1, 9, 14, 5), SampleDesc(0, 0, 0, 33), SampleDesc(1, 11, 13, 2)]
    w = make_random_pack(980, S=3, H=2, D=128, rope_axes=2, descs=descs)
    got, ref, pack = _run(w, 512, 981)
    _check_all(got, ref, pack, "small")


def test_mmdit_block_bwd_image_only_3d():
    """No text token anywhere: the text weights' gradients are exactly zero;
    3D RoPE, head_dim 64."""
    descs = [SampleDesc(2, 6, 7, 0), SampleDesc(2, 5, 9, 0)]
    w = make_random_pack(982, S=2, H=4, D=64, rope_axes=3, descs=descs)
    got, ref, pack = _run(w, 256, 983)
    for n in ("Wq", "Wk", "Wv", "Wo", "Wup", "Wdown"):
        assert np.all(got[n][1] == 0.0), f"d{n}[1] must be zero without text tokens"
    _check_all(got, ref, pack, "image-only")


def test_mmdit_block_bwd_medium_pack():
    """~1900 tokens over three samples: several tiles per sample, ragged ends,
    hid 256, MLP width 1024."""
    descs = [SampleDesc(1, 32, 40, 70), SampleDesc(1, 20, 20, 9), SampleDesc(0, 0, 0, 130)]
    w = make_random_pack(984, S=3, H=2, D=128, rope_axes=2, descs=descs)
    got, ref, pack = _run(w, 1024, 985)
    _check_all(got, ref, pack, "medium")


def test_mmdit_block_bwd_wide_layers():
    """hid 1024 (8 heads x 128) and MLP width 4096: every linear product runs
    over several 256-column tiles and K steps; ~660 tokens, 3D RoPE."""
    descs = [SampleDesc(2, 12, 16, 40), SampleDesc(1, 14, 18, 6)]
    w = make_random_pack(986, S=2, H=8, D=128, rope_axes=3, descs=descs)
    got, ref, pack = _run(w, 4096, 987)
    _check_all(got, ref, pack, "wide")
