"""The Mage-VAE conv block's kernels on the GPU through the C ABI against the
float64 oracle (``oracle/vae_oracle.py``) on the same seeded inputs: the 3x3
convolution (implicit GEMM on tcgen05, bias and residual in the epilogue) on
ragged images whose pixel tiles overhang the edges, both output-channel tile
widths and a one-row image; SiLU(GroupNorm) (deterministic statistics); and
the whole block in full on a small image, at a decoder-stage size, with one
group of 512 channels (wider than the conv's channel tile) and with two groups.

Tolerances: a conv or GroupNorm output is one bf16 rounding of an fp32 result
(max-abs 2e-2, relative RMS 5e-3, as for the attention path); the block adds
bf16-stored intermediates that the GPU and the oracle round independently, so
its bound is 2e-2 plus one bf16 ulp at the value's magnitude (gpu_util)."""

import numpy as np
import pytest
import torch

import oracle
from packgen import make_vae_block

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import resolution_packed_diffusion_b200 as mf  # noqa: E402
from gpu_util import assert_bf16_close, assert_block_close, dev_bf16, host_f32  # noqa: E402


@pytest.fixture(params=[0, 1], ids=["one_cta", "cta_pair"])
def conv_pair(request):
    """Both conv kernels: one CTA per 128-pixel tile, and CTA pairs computing two
    vertically adjacent tiles as M = 256 MMAs (the second tile may lie wholly
    below the image)."""
    mf.mf_set_conv_cta_pair(request.param)
    yield request.param
    mf.mf_set_conv_cta_pair(0)  # the library's default


def _f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _conv_case(N, H, W, Cin, Cout, seed, bias=True, residual=True):
    rng = np.random.default_rng(seed)
    from packgen import f32_to_bf16_bits
    xb = f32_to_bf16_bits(rng.standard_normal((N, H, W, Cin), dtype=np.float32))
    wb = f32_to_bf16_bits((rng.standard_normal((Cout, 3, 3, Cin), dtype=np.float32)
                           / np.float32(np.sqrt(9.0 * Cin))).astype(np.float32))
    b = (0.1 * rng.standard_normal(Cout)).astype(np.float32) if bias else None
    rb = f32_to_bf16_bits(rng.standard_normal((N, H, W, Cout), dtype=np.float32)) if residual \
        else None
    x, Wt = dev_bf16(xb), dev_bf16(wb)
    y = torch.empty((N, H, W, Cout), dtype=torch.bfloat16, device="cuda")
    mf.mf_conv3x3(x, Wt, _f32(b) if bias else None, dev_bf16(rb) if residual else None, N, H, W,
                  Cin, Cout, y)
    assert mf.mf_get_error() == mf.MF_OK
    from packgen import bf16_bits_to_f32
    ref = oracle.conv3x3(bf16_bits_to_f32(xb), bf16_bits_to_f32(wb), b,
                         bf16_bits_to_f32(rb) if residual else None)
    return host_f32(y), ref


@pytest.mark.parametrize("N,H,W,Cin,Cout,bias,residual", [
    (2, 9, 13, 64, 128, True, True),      # 16 x 8 pixel tiles overhanging both edges
    (2, 9, 13, 64, 128, False, False),
    (1, 17, 33, 128, 256, True, False),   # 256 output channels per tile
    (1, 1, 200, 64, 64, True, True),      # one image row: every tap above and below reads zeros
    (3, 40, 24, 256, 128, False, True),   # four channel blocks per tap
], ids=["ragged", "ragged_plain", "n256", "one_row", "cin256"])
@pytest.mark.usefixtures("conv_pair")
def test_conv3x3(N, H, W, Cin, Cout, bias, residual):
    got, ref = _conv_case(N, H, W, Cin, Cout, 5000 + H * W + Cin, bias, residual)
    assert_bf16_close(got, ref, "conv3x3")


@pytest.mark.parametrize("N,H,W,C,G", [(2, 9, 13, 64, 8), (1, 31, 17, 256, 32),
                                       (2, 64, 64, 128, 16)])
def test_group_norm_silu(N, H, W, C, G):
    v = make_vae_block(N=N, H=H, W=W, C=C, G=G, seed=5100 + C)
    x = dev_bf16(v.x_bits)
    # a mean far from zero checks the statistics' cancellation behaviour
    x = (x.float() * 0.5 + 3.0).to(torch.bfloat16)
    ws_bytes = mf.mf_gn_workspace_size(N, H, W, G)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        y = torch.empty_like(x)
        mf.mf_group_norm_silu(x, _f32(v.gamma1), _f32(v.beta1), N, H, W, C, G, v.eps, y, ws,
                              ws_bytes)
        assert mf.mf_get_error() == mf.MF_OK
        outs.append(y)
    assert torch.equal(outs[0], outs[1]), "statistics are merged in a fixed order"
    ref = oracle.group_norm_silu(host_f32(x), v.gamma1, v.beta1, G, v.eps)
    assert_bf16_close(host_f32(outs[0]), ref, "SiLU(GroupNorm)")


def _block(v):
    dv = {k: dev_bf16(getattr(v, k + "_bits")) for k in ("x", "W1", "W2")}
    fv = {k: _f32(getattr(v, k)) for k in ("gamma1", "beta1", "gamma2", "beta2", "c1", "c2")}
    y = torch.empty_like(dv["x"])
    ws_bytes = mf.mf_vae_block_workspace_size(v.N, v.H, v.W, v.C, v.G)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    mf.mf_vae_res_block(dv["x"], fv["gamma1"], fv["beta1"], dv["W1"], fv["c1"], fv["gamma2"],
                        fv["beta2"], dv["W2"], fv["c2"], v.N, v.H, v.W, v.C, v.G, v.eps, y, ws,
                        ws_bytes)
    assert mf.mf_get_error() == mf.MF_OK
    return host_f32(y)


@pytest.mark.parametrize("name,shape", [
    ("tiny", None),
    ("stage_1_8", None),
    # one group of 512 channels: wider than the conv's 256-channel tile
    (None, dict(N=1, H=6, W=7, C=512, G=1)),
    # two groups of 64 channels
    (None, dict(N=2, H=11, W=5, C=128, G=2)),
], ids=["tiny", "stage_1_8", "one_group_512ch", "two_groups"])
@pytest.mark.usefixtures("conv_pair")
def test_vae_res_block(name, shape):
    v = make_vae_block(name, **(shape or {}))
    got = _block(v)
    ref = oracle.vae_res_block(v.f32("x"), v.gamma1, v.beta1, v.f32("W1"), v.c1, v.gamma2,
                               v.beta2, v.f32("W2"), v.c2, v.G, v.eps)
    assert_block_close(got, ref, f"VAE block ({name})")


def test_conv_pair_setting_is_checked():
    with pytest.raises(mf.MFError):
        mf.mf_set_conv_cta_pair(2)


def test_vae_entry_points_reject_bad_arguments():
    x = torch.zeros((1, 4, 4, 64), dtype=torch.bfloat16, device="cuda")
    Wt = torch.zeros((64, 3, 3, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mf.MFError):  # y overlaps x
        mf.mf_conv3x3(x, Wt, None, None, 1, 4, 4, 64, 64, x)
    with pytest.raises(mf.MFError):  # 96 channels: not a supported width
        mf.mf_conv3x3(x, Wt, None, None, 1, 4, 4, 96, 64, torch.empty_like(x))
    ws = torch.empty(mf.mf_gn_workspace_size(1, 4, 4, 8), dtype=torch.uint8, device="cuda")
    g = torch.ones(64, device="cuda")
    with pytest.raises(mf.MFError):  # 64 / 16 = 4 channels a group: not a multiple of 8
        mf.mf_group_norm_silu(x, g, g, 1, 4, 4, 64, 16, 1e-6, torch.empty_like(x), ws, ws.numel())
    assert mf.mf_get_error() == mf.MF_OK
