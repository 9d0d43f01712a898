"""Packed classifier-free guidance on the GPU, through the C ABI, against the
oracle (picx.dev "Mage-Flow" summary, Methodology > NR-MMDiT, "Packed CFG
inference": both branches of an image are samples of one pack)."""

import numpy as np
import pytest
import torch

import oracle
import resolution_packed_diffusion_b200 as mf
from gpu_util import DevicePack, assert_bf16_close, dev_bf16, host_f32
from packgen import SampleDesc, f32_to_bf16_bits, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def test_cfg_combine_on_the_block_output():
    """The packed-CFG workload: the block's output y of both branches, guided
    at w = 4.5 over the 4096 image tokens."""
    w = make_workload(3)
    dp = DevicePack(w)
    _, y = dp.block()
    assert mf.mf_get_error() == mf.MF_OK
    n_img = 64 * 64
    out = torch.empty((n_img, w.hid), dtype=torch.bfloat16, device="cuda")
    mf.mf_cfg_combine(y, w.descs, w.cfg_pairs, w.hid, 4.5, out)
    assert mf.mf_get_error() == mf.MF_OK
    ref = oracle.cfg_combine(host_f32(y), w.descs, w.cfg_pairs, 4.5)
    assert_bf16_close(host_f32(out), ref, "guided output")


DESCS = [SampleDesc(1, 9, 14, 5), SampleDesc(0, 0, 0, 33), SampleDesc(1, 14, 9, 2),
         SampleDesc(1, 3, 3, 1), SampleDesc(1, 1, 9, 60), SampleDesc(2, 0, 5, 4)]
PAIRS = [(0, 2), (4, 3), (2, 0)]  # 126, 9 and 126 image tokens; the last swaps roles


@pytest.mark.parametrize("wv", [0.0, 1.0, -1.5, 7.25])
def test_cfg_combine_pairs(wv):
    C = 64
    T = sum(d.frames * d.grid_h * d.grid_w + d.n_text for d in DESCS)
    rng = np.random.default_rng(90)
    bits = f32_to_bf16_bits(rng.standard_normal((T, C), dtype=np.float32))
    v = dev_bf16(bits)
    rows = 126 + 9 + 126
    out = torch.empty((rows, C), dtype=torch.bfloat16, device="cuda")
    mf.mf_cfg_combine(v, DESCS, PAIRS, C, wv, out)
    assert mf.mf_get_error() == mf.MF_OK
    ref = oracle.cfg_combine(host_f32(v), DESCS, PAIRS, wv)
    got = host_f32(out)
    assert_bf16_close(got, ref, f"guided output at w={wv}")
    if wv == 0.0:  # fma(0, c - u, u) is u exactly
        assert np.array_equal(got, ref)


def test_cfg_combine_rejects_bad_pairs():
    C = 64
    T = sum(d.frames * d.grid_h * d.grid_w + d.n_text for d in DESCS)
    v = torch.zeros((T, C), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((300, C), dtype=torch.bfloat16, device="cuda")
    for pairs in ([(0, 3)], [(1, 1)], [(0, 9)]):  # grids differ, same sample, out of range
        with pytest.raises(mf.MFError) as e:
            mf.mf_cfg_combine(v, DESCS, pairs, C, 2.0, out)
        assert e.value.status == mf.MF_ERR_INVALID
    with pytest.raises(mf.MFError):
        mf.mf_cfg_combine(v, DESCS, PAIRS, 60, 2.0, out)  # C not a multiple of 8
    with pytest.raises(mf.MFError):
        mf.mf_cfg_combine(v, DESCS, PAIRS, C, float("nan"), out)
    assert torch.count_nonzero(out).item() == 0  # nothing was launched
