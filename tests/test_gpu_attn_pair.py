"""The attention on CTA pairs (mf_set_attn_cta_pair(1): thread-block clusters of
two CTAs whose tensor cores run each QK^T and PV product as one M = 256 tcgen05
MMA, each CTA holding half of every K and V tile) against the float64 oracle,
through the C ABI: the workloads at full size (block forward with RoPE in the Q
prologue, attention with and without RoPE, the LSE), edge packs whose 512-row
work items leave one CTA of the pair or the whole second tile without a valid
row, both work orders, and the online-softmax stress case. Same tolerances as
the one-CTA kernel (max-abs 2e-2, relative RMS 5e-3)."""

import math

import numpy as np
import pytest
import torch

import oracle
from packgen import SampleDesc, make_random_pack, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import resolution_packed_diffusion_b200 as mf  # noqa: E402
from gpu_util import DevicePack, assert_bf16_close, host_f32, oracle_pack, sample_rows  # noqa: E402


@pytest.fixture(autouse=True)
def cta_pairs():
    mf.mf_set_attn_cta_pair(1)
    yield
    mf.mf_set_attn_cta_pair(0)


def _check_block(w, rows=None):
    dp = DevicePack(w)
    pack = oracle_pack(w)
    mod = oracle.adaln_params(w.c, w.W, w.hid)
    x_mod, y = dp.block()
    assert mf.mf_get_error() == mf.MF_OK
    ref_xm, ref_y, _ = oracle.block_fwd(w.f32("x"), w.f32("q"), w.f32("k"), w.f32("v"), mod, pack,
                                        w.rope_axes, w.base, w.eps, rows=rows)
    sel = slice(None) if rows is None else rows
    assert_bf16_close(host_f32(x_mod)[sel], ref_xm, "pair block x_mod")
    assert_bf16_close(host_f32(y)[sel], ref_y, "pair block y")
    return dp, pack


@pytest.mark.parametrize("idx", [2, 3, 4, 5],
                         ids=["training_pack", "cfg_pack", "edit_pack", "large_pack"])
def test_pair_block_and_attention_full_size(idx):
    w = make_workload(idx)
    pack = oracle_pack(w)
    rows = sample_rows(pack["cu_seqlens"], 24, 3000 + idx)
    dp, pack = _check_block(w, rows)
    # plain attention on the unrotated inputs (no RoPE), with the LSE
    o, lse = dp.attention(dp.q, dp.k, dp.v, with_rope=False, lse=True)
    assert mf.mf_get_error() == mf.MF_OK
    ref_o, ref_lse = oracle.varlen_attention(w.f32("q"), w.f32("k"), w.f32("v"),
                                             pack["cu_seqlens"], rows=rows)
    assert_bf16_close(host_f32(o)[rows], ref_o, "pair attention O")
    assert np.abs(lse.cpu().numpy()[:, rows].astype(np.float64) - ref_lse).max() <= 2e-2
    # deterministic: a second block forward gives the same bits
    x1, y1 = dp.block()
    x2, y2 = dp.block()
    assert torch.equal(x1, x2) and torch.equal(y1, y2)


PAIR_EDGE_PACKS = [
    # (descs, H, axes): D = 128 throughout (the pair kernel's head size)
    ([SampleDesc(0, 0, 0, 1)], 1, 2),                                          # one token
    ([SampleDesc(1, 10, 10, 0), SampleDesc(1, 3, 3, 1)], 2, 2),                # 100 and 10 rows: rank 1 idle
    ([SampleDesc(1, 15, 20, 0), SampleDesc(1, 1, 1, 199)], 2, 2),              # 300 and 200 rows
    ([SampleDesc(1, 1, 127, 0), SampleDesc(1, 8, 16, 0), SampleDesc(1, 1, 129, 0)], 2, 2),
    ([SampleDesc(0, 0, 0, 700), SampleDesc(1, 5, 7, 3)], 3, 2),                # text-only, 700 rows
    ([SampleDesc(1, 4, 4, 0), SampleDesc(0, 0, 0, 0), SampleDesc(1, 3, 3, 5)], 2, 2),  # empty
    ([SampleDesc(2, 6, 5, 7), SampleDesc(1, 9, 4, 2), SampleDesc(2, 3, 3, 0)], 2, 3),  # 3D
    ([SampleDesc(1, 16, 32, 0), SampleDesc(1, 16, 32, 1)], 2, 2),              # 512 and 513 rows
    ([SampleDesc(1, 16, 48, 255)], 1, 2),                                      # 1023 rows
]


@pytest.mark.parametrize("k", range(len(PAIR_EDGE_PACKS)))
def test_pair_edge_packs_full_compare(k):
    descs, H, axes = PAIR_EDGE_PACKS[k]
    w = make_random_pack(3100 + k, S=len(descs), H=H, D=128, rope_axes=axes, descs=descs)
    dp, pack = _check_block(w)
    o, lse = dp.attention(dp.q, dp.k, dp.v, with_rope=False, lse=True)
    assert mf.mf_get_error() == mf.MF_OK
    ref_o, ref_lse = oracle.varlen_attention(w.f32("q"), w.f32("k"), w.f32("v"),
                                             pack["cu_seqlens"])
    assert_bf16_close(host_f32(o), ref_o, "pair edge O")
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 2e-2
    o2, _ = dp.attention(dp.q, dp.k, dp.v, with_rope=True)
    assert mf.mf_get_error() == mf.MF_OK
    q_r = oracle.rope_apply(w.f32("q"), pack["pos_ids"], axes)
    k_r = oracle.rope_apply(w.f32("k"), pack["pos_ids"], axes)
    ref_o2, _ = oracle.varlen_attention(q_r, k_r, w.f32("v"), pack["cu_seqlens"])
    assert_bf16_close(host_f32(o2), ref_o2, "pair edge O (RoPE)")


@pytest.mark.parametrize("descs,H", [
    ([SampleDesc(1, 64, 64, 0), SampleDesc(1, 40, 40, 100), SampleDesc(1, 24, 24, 10),
      SampleDesc(1, 10, 10, 5), SampleDesc(0, 0, 0, 77)], 8),              # unequal items
    ([SampleDesc(1, 32, 32, 0)] * 4, 16),                                   # equal items
], ids=["unequal", "equal"])
def test_pair_work_orders(descs, H):
    """Every item is covered once whichever work order the launch picks for the
    pairs (host greedy table or in-kernel snake deal)."""
    w = make_random_pack(3200 + H, S=len(descs), H=H, D=128, rope_axes=2, descs=descs)
    dp = DevicePack(w)
    pack = oracle_pack(w)
    o, _ = dp.attention(dp.q, dp.k, dp.v, with_rope=False)
    assert mf.mf_get_error() == mf.MF_OK
    rows = sample_rows(pack["cu_seqlens"], 8, 3200 + H)
    ref_o, _ = oracle.varlen_attention(w.f32("q"), w.f32("k"), w.f32("v"), pack["cu_seqlens"],
                                       rows=rows)
    assert_bf16_close(host_f32(o)[rows], ref_o, "pair attention O")


@pytest.mark.parametrize("step", [29.0, 3.0], ids=["jumps", "creeps"])
def test_pair_when_the_row_max_keeps_growing(step):
    """As for the one-CTA kernel: scores that climb by `step` log2 units per
    128-key tile for some rows (29 forces the reference max to move), fall for
    others; head_dim 128, so both CTAs of a pair hold such rows."""
    from packgen import f32_to_bf16_bits
    descs = [SampleDesc(1, 24, 25, 0), SampleDesc(1, 7, 9, 3)]  # 600 and 66 tokens
    H, D = 2, 128
    w = make_random_pack(3300, S=len(descs), H=H, D=D, rope_axes=2, descs=descs)
    rng = np.random.default_rng(3301)
    T = w.T
    u = np.full(D, 1.0 / math.sqrt(D))  # |u|^2 = 1
    a = rng.choice([4.0, -4.0, 0.5], size=(T, H))
    tile = (np.arange(T) % 600) // 128
    # x = s * log2(e) / sqrt(D) = a * b * log2(e) / sqrt(D): b rises by step per tile
    b = 1.0 + tile * step * math.sqrt(D) / (4.0 * 1.4426950408889634)
    q = a[:, :, None] * u + 0.05 * rng.standard_normal((T, H, D))
    k = b[:, None, None] * u + 0.05 * rng.standard_normal((T, H, D))
    w.q_bits = f32_to_bf16_bits(q.astype(np.float32))
    w.k_bits = f32_to_bf16_bits(k.astype(np.float32))
    dp = DevicePack(w)
    pack = oracle_pack(w)
    o, lse = dp.attention(dp.q, dp.k, dp.v, with_rope=False, lse=True)
    assert mf.mf_get_error() == mf.MF_OK
    ref_o, ref_lse = oracle.varlen_attention(w.f32("q"), w.f32("k"), w.f32("v"), pack["cu_seqlens"])
    assert_bf16_close(host_f32(o), ref_o, "pair attention O")
    assert np.all(np.abs(lse.cpu().numpy() - ref_lse) <= 2e-2 * np.maximum(1.0, np.abs(ref_lse) / 8))


def test_pair_setting_is_checked_and_per_device():
    with pytest.raises(mf.MFError):
        mf.mf_set_attn_cta_pair(2)
    mf.mf_set_attn_cta_pair(0)
    mf.mf_set_attn_cta_pair(1)
