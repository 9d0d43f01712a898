"""The modality-specific linear layer on the GPU (tcgen05), through the C ABI,
against the oracle: every row of small packs whose 128-row tiles mix image and
text tokens, and sampled rows of a full-size projection. Each case runs on both
kernels: one CTA per 128-row tile, and CTA pairs (mf_set_linear_cta_pair(1),
256-row tiles as M = 256 MMAs over two SMs, whose row blocks may hold a
modality in one CTA's half only)."""

import numpy as np
import pytest
import torch

import oracle
import resolution_packed_diffusion_b200 as mf
from gpu_util import assert_bf16_close, dev_bf16, host_f32, sample_rows
from packgen import SampleDesc, f32_to_bf16_bits, make_random_pack, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


@pytest.fixture(params=[0, 1], ids=["one_cta", "cta_pair"], autouse=True)
def cta_pair(request):
    mf.mf_set_linear_cta_pair(request.param)
    yield request.param
    mf.mf_set_linear_cta_pair(1)  # the library's default


def _run(descs, K, N, seed, act=0):
    rng = np.random.default_rng(seed)
    pack = oracle.pack_build(descs, 2)
    T = pack["T"]
    x_bits = f32_to_bf16_bits(rng.standard_normal((T, K), dtype=np.float32))
    w_bits = f32_to_bf16_bits((rng.standard_normal((2, N, K), dtype=np.float32)
                               / np.float32(np.sqrt(K))).astype(np.float32))
    x, W = dev_bf16(x_bits), dev_bf16(w_bits)
    tm = torch.from_numpy(pack["tok_mod"]).cuda()
    out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    mf.mf_modality_linear(x, W, tm, descs, K, N, out, act)
    assert mf.mf_get_error() == mf.MF_OK
    return pack, host_f32(x), host_f32(W), host_f32(out)


SMALL = [
    ([SampleDesc(1, 9, 14, 5), SampleDesc(0, 0, 0, 33), SampleDesc(1, 14, 9, 2),
      SampleDesc(1, 3, 3, 1), SampleDesc(1, 1, 9, 60)], 128, 256),
    ([SampleDesc(1, 16, 16, 20), SampleDesc(1, 8, 32, 12)], 192, 512),   # the 544-token pack
    ([SampleDesc(1, 1, 1, 0)], 64, 256),                                  # one token
    ([SampleDesc(0, 0, 0, 300), SampleDesc(1, 11, 13, 0)], 320, 256),    # text-only sample
    # a 256-row block whose first 128 rows are image and second 128 rows text:
    # each modality lives in one CTA's half of the pair's block
    ([SampleDesc(1, 8, 16, 128), SampleDesc(1, 16, 8, 128)], 128, 256),
]


@pytest.mark.parametrize("k", range(len(SMALL)))
def test_linear_every_row(k):
    descs, K, N = SMALL[k]
    pack, x, W, out = _run(descs, K, N, 900 + k)
    ref = oracle.modality_linear(x, W, pack["tok_mod"])
    assert np.isfinite(out).all()
    assert_bf16_close(out, ref, "linear out")


@pytest.mark.parametrize("k", [0, 1])
def test_linear_gelu_every_row(k):
    descs, K, N = SMALL[k]
    pack, x, W, out = _run(descs, K, N, 920 + k, act=mf.MF_ACT_GELU)
    ref = oracle.modality_linear(x, W, pack["tok_mod"], "gelu")
    assert np.isfinite(out).all()
    assert_bf16_close(out, ref, "linear + GELU out")


def test_linear_qkv_projection_of_the_training_pack():
    """Full size: the training pack's 16384 tokens through a 3072 -> 9216
    projection (the fused Q, K, V widths), rows sampled around every sample and
    tile boundary."""
    w = make_workload(2, with_arrays=False)
    pack, x, W, out = _run(w.descs, 3072, 9216, 950)
    rows = sample_rows(pack["cu_seqlens"], 64, 951)
    ref = oracle.modality_linear(x[rows], W, pack["tok_mod"][rows])
    assert np.isfinite(out).all()
    assert_bf16_close(out[rows], ref, "projection rows")


def test_linear_pair_setting_is_checked():
    with pytest.raises(mf.MFError):
        mf.mf_set_linear_cta_pair(2)


def test_linear_rejects_bad_shapes():
    descs = [SampleDesc(1, 4, 4, 3)]
    x = torch.zeros((19, 128), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((2, 256, 128), dtype=torch.bfloat16, device="cuda")
    tm = torch.zeros(19, dtype=torch.uint8, device="cuda")
    out = torch.zeros((19, 256), dtype=torch.bfloat16, device="cuda")
    for K, N, act in ((96, 256, 0), (128, 200, 0), (128, 256, 2)):
        with pytest.raises(mf.MFError) as e:
            mf.mf_modality_linear(x, W, tm, descs, K, N, out, act)
        assert e.value.status == mf.MF_ERR_INVALID
    with pytest.raises(mf.MFError):
        mf.mf_modality_linear(x, W, tm, descs, 128, 256, x)  # out overlaps x
