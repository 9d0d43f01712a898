"""mf_block_fwd_noalloc: the block forward for callers that cannot allocate
device memory (a plugin whose host application owns all device memory, or a
caller that must not make a call which can synchronise the device). It keeps the
rotated Q and K in the library's own fixed device array instead of a
caller-provided workspace.

Checked through the C ABI on two calls in a row against mf_block_fwd (which
takes a workspace) and against the float64 oracle, with the tolerance the parity
tests use. This file is collected last on purpose and needs nothing from the
other test files."""

import numpy as np
import pytest
import torch

import oracle
from packgen import SampleDesc, make_random_pack, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import resolution_packed_diffusion_b200 as mf  # noqa: E402
from gpu_util import DevicePack, assert_bf16_close, host_f32, oracle_pack  # noqa: E402


def _noalloc(dp):
    x_mod = torch.empty((dp.T, dp.hid), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((dp.T, dp.hid), dtype=torch.bfloat16, device="cuda")
    mf.mf_block_fwd_noalloc(dp.x, dp.q, dp.k, dp.v, dp.mod, dp.cu_d, dp.cu_h, dp.pos,
                            dp.tok_sample, dp.tok_mod, dp.S, dp.H, dp.D, dp.w.rope_axes,
                            dp.w.base, dp.w.eps, x_mod, y)
    return x_mod, y


PACKS = [
    ("544-token pack, 2 x 64", lambda: make_workload(1)),
    ("2404-token pack, 24 x 128",
     lambda: make_random_pack(900, S=2, H=24, D=128, rope_axes=2,
                              descs=[SampleDesc(1, 48, 48, 100), SampleDesc(0, 0, 0, 0)])),
    ("edit pack, 3D RoPE, 8 x 128",
     lambda: make_random_pack(901, S=2, H=8, D=128, rope_axes=3,
                              descs=[SampleDesc(2, 20, 24, 33), SampleDesc(1, 17, 9, 5)])),
]


@pytest.mark.parametrize("name,make", PACKS, ids=[p[0] for p in PACKS])
def test_noalloc_matches_workspace_entry_point_twice(name, make):
    w = make()
    dp = DevicePack(w)
    ref_xm, ref_y = dp.block()
    assert mf.mf_get_error() == mf.MF_OK
    ref_xm, ref_y = host_f32(ref_xm), host_f32(ref_y)
    mod = oracle.adaln_params(w.c, w.W, w.hid)
    o_xm, o_y, _ = oracle.block_fwd(w.f32("x"), w.f32("q"), w.f32("k"), w.f32("v"), mod,
                                    oracle_pack(w), w.rope_axes, w.base, w.eps)
    for call in range(2):  # the array keeps the previous call's contents
        x_mod, y = _noalloc(dp)
        assert mf.mf_get_error() == mf.MF_OK
        x_mod, y = host_f32(x_mod), host_f32(y)
        assert_bf16_close(x_mod, ref_xm, f"{name}: x_mod vs mf_block_fwd, call {call}")
        assert_bf16_close(y, ref_y, f"{name}: y vs mf_block_fwd, call {call}")
        assert_bf16_close(x_mod, o_xm, f"{name}: x_mod vs oracle, call {call}")
        assert_bf16_close(y, o_y, f"{name}: y vs oracle, call {call}")


def test_noalloc_rejects_a_pack_beyond_its_array():
    w = make_workload(2, with_arrays=False)  # 16384 tokens need ~105 MB: rotated k and table
    cu_h, T = mf.mf_pack_build(w.descs, w.rope_axes, w.budget)
    assert mf.mf_workspace_size(T, w.H, w.D, 1) > mf.MF_NOALLOC_SCRATCH_BYTES
    st = mf.lib.mf_block_fwd_noalloc(16, 16, 16, 16, 16, 16, cu_h.ctypes.data, 16, 16, 16,
                                     w.S, w.H, w.D, 2, 10000.0, 1e-6, 16, 16, None)
    assert st == mf.MF_ERR_UNSUPPORTED
