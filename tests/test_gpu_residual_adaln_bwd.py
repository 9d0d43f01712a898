"""Backward of the gated residual (mf_gated_residual_bwd) and of the adaLN
modulation (mf_adaln_modulate_bwd), through the C ABI, against the float64
oracle on the same seeded inputs: small packs with empty samples and image /
text boundaries in full, and the training pack at full size.

Tolerances: bf16 outputs (dO, dx) follow the block's rule (max-abs 2e-2,
relative RMS 5e-3). The per-(sample, modality) sums are fp32: rows are summed
in chunks of 64 and the chunk sums added with atomics, so by the recursive
summation bound each sum is within about 128 * 2^-24 of the sum of its terms'
magnitudes; the x-hat inside dscale carries the fp32 error of the row
statistics (a few 2^-24 times the row length's share per lane, under 1e-5
relative). The tests allow 3e-5 times the sum of |terms|, plus 1e-6. Slots a
call must not write are pre-filled with a sentinel and must keep it.
"""

import numpy as np
import pytest
import torch

import oracle
from packgen import SampleDesc, draw_grad_bits, make_random_pack, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import resolution_packed_diffusion_b200 as mf  # noqa: E402
from gpu_util import DevicePack, assert_bf16_close, dev_bf16, host_f32, oracle_pack  # noqa: E402
from packgen import bf16_bits_to_f32  # noqa: E402

SENTINEL = 7.0
SUM_REL = 3e-5

PACKS = [
    # (descs, H, D)
    ([SampleDesc(1, 9, 9, 40), SampleDesc(0, 0, 0, 0), SampleDesc(1, 7, 11, 3),
      SampleDesc(1, 4, 4, 0)], 2, 64),
    ([SampleDesc(1, 16, 16, 20), SampleDesc(1, 8, 32, 12)], 2, 64),
    ([SampleDesc(1, 12, 20, 33), SampleDesc(0, 0, 0, 5)], 3, 128),
]


def assert_sums_close(got, ref, mag, name):
    err = np.abs(got - ref)
    tol = SUM_REL * mag + 1e-6
    worst = int(np.argmax(err - tol))
    assert (err <= tol).all(), (f"{name}: |err| {err.flat[worst]:.3g} > {tol.flat[worst]:.3g} "
                                f"at {np.unravel_index(worst, err.shape)}")


def seg_abs_sums(vals, ts, tm, S):
    """Per-(sample, modality) sums of |vals| (the magnitude scale of each sum)."""
    out = np.zeros((S, 2, vals.shape[1]))
    np.add.at(out, (ts.astype(np.int64), tm.astype(np.int64)), np.abs(vals))
    return out


def run_gate(w, mod, seed):
    dp = DevicePack(w)
    pack = oracle_pack(w)
    T, S, hid = w.T, w.S, w.hid
    dy_bits = draw_grad_bits(seed, (T, hid))
    o_bits = draw_grad_bits(seed + 1, (T, hid))
    dy, o = dev_bf16(dy_bits), dev_bf16(o_bits)
    mod_d = torch.from_numpy(mod.astype(np.float32)).cuda()
    dmod = torch.full((S, 2, 3, hid), SENTINEL, dtype=torch.float32, device="cuda")
    d_o = torch.empty_like(dy)
    mf.mf_gated_residual_bwd(dy, o, mod_d, dp.tok_sample, dp.tok_mod, T, S, hid, d_o, dmod)
    assert mf.mf_get_error() == mf.MF_OK
    ts, tm = pack["tok_sample"], pack["tok_mod"]
    fdy, fo = bf16_bits_to_f32(dy_bits), bf16_bits_to_f32(o_bits)
    mod32 = mod.astype(np.float32).astype(np.float64)
    _, r_do, r_dmod = oracle.gated_residual_bwd(fdy, fo, mod32, ts, tm, S)
    assert_bf16_close(host_f32(d_o), r_do, "gate backward dO")
    got = dmod.cpu().numpy().astype(np.float64)
    assert_sums_close(got[:, :, 2], r_dmod[:, :, 2], seg_abs_sums(fdy * fo, ts, tm, S), "dgate")
    assert (got[:, :, :2] == SENTINEL).all(), "shift / scale slots were written"


def run_adaln(w, mod, seed, with_resid):
    dp = DevicePack(w)
    pack = oracle_pack(w)
    T, S, hid = w.T, w.S, w.hid
    g_bits = draw_grad_bits(seed, (T, hid))
    r_bits = draw_grad_bits(seed + 1, (T, hid))
    dxm = dev_bf16(g_bits)
    resid = dev_bf16(r_bits) if with_resid else None
    mod_d = torch.from_numpy(mod.astype(np.float32)).cuda()
    dmod = torch.full((S, 2, 3, hid), SENTINEL, dtype=torch.float32, device="cuda")
    dx = resid if with_resid else torch.empty_like(dxm)  # in place over resid
    ws_bytes = mf.mf_adaln_bwd_workspace_size(T)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    mf.mf_adaln_modulate_bwd(dxm, dp.x, mod_d, dp.tok_sample, dp.tok_mod, resid, T, S, hid,
                             w.eps, dx, dmod, ws, ws_bytes)
    assert mf.mf_get_error() == mf.MF_OK
    ts, tm = pack["tok_sample"], pack["tok_mod"]
    fg, fx = bf16_bits_to_f32(g_bits), w.f32("x")
    mod32 = mod.astype(np.float32).astype(np.float64)
    r_dx, r_dmod = oracle.adaln_modulate_bwd(fg, fx, mod32, ts, tm, S, w.eps)
    if with_resid:
        r_dx = r_dx + bf16_bits_to_f32(r_bits)
    assert_bf16_close(host_f32(dx), r_dx, "adaLN backward dx")
    got = dmod.cpu().numpy().astype(np.float64)
    xhat = oracle.layer_norm_rows(fx, w.eps)
    assert_sums_close(got[:, :, 0], r_dmod[:, :, 0], seg_abs_sums(fg, ts, tm, S), "dshift")
    assert_sums_close(got[:, :, 1], r_dmod[:, :, 1], seg_abs_sums(fg * xhat, ts, tm, S),
                      "dscale")
    assert (got[:, :, 2] == SENTINEL).all(), "gate slots were written"


def small_case(k):
    descs, H, D = PACKS[k]
    w = make_random_pack(1500 + k, S=len(descs), H=H, D=D, rope_axes=2, descs=descs)
    mod = 0.3 * np.random.default_rng(1600 + k).standard_normal((w.S, 2, 3, w.hid))
    return w, mod


@pytest.mark.parametrize("k", range(len(PACKS)))
def test_gate_bwd_small_packs(k):
    w, mod = small_case(k)
    run_gate(w, mod, 1700 + k)


@pytest.mark.parametrize("k", range(len(PACKS)))
@pytest.mark.parametrize("with_resid", [False, True], ids=["plain", "resid_in_place"])
def test_adaln_bwd_small_packs(k, with_resid):
    w, mod = small_case(k)
    run_adaln(w, mod, 1800 + k, with_resid)


def test_gate_and_adaln_bwd_training_pack():
    w = make_workload(2)
    mod = oracle.adaln_params(w.c, w.W, w.hid)
    run_gate(w, mod, 1900)
    run_adaln(w, mod, 1910, True)


@pytest.mark.parametrize("S,C,hid", [(5, 128, 3072), (11, 40, 136), (1, 1, 8)],
                         ids=["training_pack_shape", "several_sample_passes", "minimal"])
def test_adaln_params_bwd(S, C, hid):
    """The modulation map's backward (mf_adaln_params_bwd): dc = dmod W^T and
    dW = c^T dmod against the oracle, fp32 sums within 3e-5 of the sum of their
    terms' magnitudes; twice in a row with the same bits (no atomics)."""
    rng = np.random.default_rng(2300 + S)
    c = rng.standard_normal((S, C)).astype(np.float32)
    W = (0.02 * rng.standard_normal((C, 6 * hid))).astype(np.float32)
    dmod = rng.standard_normal((S, 2, 3, hid)).astype(np.float32)
    c_d, W_d, dm_d = (torch.from_numpy(a).cuda() for a in (c, W, dmod))
    outs = []
    for _ in range(2):
        dc = torch.full((S, C), SENTINEL, dtype=torch.float32, device="cuda")
        dW = torch.full((C, 6 * hid), SENTINEL, dtype=torch.float32, device="cuda")
        mf.mf_adaln_params_bwd(dm_d, c_d, W_d, S, C, hid, dc, dW)
        assert mf.mf_get_error() == mf.MF_OK
        outs.append((dc.cpu().numpy().astype(np.float64), dW.cpu().numpy().astype(np.float64)))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    r_dc, r_dW = oracle.adaln_params_bwd(dmod, c, W)
    dm = dmod.reshape(S, -1).astype(np.float64)
    mag_dc = np.abs(dm) @ np.abs(W.astype(np.float64)).T
    mag_dW = np.abs(c.astype(np.float64)).T @ np.abs(dm)
    assert_sums_close(outs[0][0], r_dc, mag_dc, "dc")
    assert_sums_close(outs[0][1], r_dW, mag_dW, "dW")
    # either output alone
    dc1 = torch.empty((S, C), dtype=torch.float32, device="cuda")
    mf.mf_adaln_params_bwd(dm_d, c_d, W_d, S, C, hid, dc1, None)
    dW1 = torch.empty((C, 6 * hid), dtype=torch.float32, device="cuda")
    mf.mf_adaln_params_bwd(dm_d, c_d, W_d, S, C, hid, None, dW1)
    assert mf.mf_get_error() == mf.MF_OK
    assert np.array_equal(dc1.cpu().numpy(), outs[0][0].astype(np.float32))
    assert np.array_equal(dW1.cpu().numpy(), outs[0][1].astype(np.float32))
