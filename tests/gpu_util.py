"""Helpers for the GPU parity tests: move seeded bf16 inputs to the device, run
the library's entry points through the C ABI, and compare with the oracle.

Comparison rule for bf16 outputs (max-abs 2e-2 and relative RMS 5e-3 against
the float64 oracle): the max-abs bound applies as stated wherever bf16 storage
can meet it (|reference| < 8, where half an ulp is at most 2^-6); where the
exact value is 8 or larger, storing it in bf16 alone can be off by up to half an
ulp (2^-5 at [8, 16)), so the bound there is 2e-2 plus that half ulp.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import resolution_packed_diffusion_b200 as mf
from packgen import Workload, bf16_bits_to_f32

MAX_ABS = 2e-2
REL_RMS = 5e-3
# gradients of the attention: relative to each tensor and sample (see
# assert_grad_close)
GRAD_REL_RMS = 5e-3
GRAD_MAX_REL = 2.0 ** -5


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_f32(t: torch.Tensor) -> np.ndarray:
    return bf16_bits_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def half_ulp_bf16(ref: np.ndarray) -> np.ndarray:
    a = np.abs(ref)
    e = np.floor(np.log2(np.maximum(a, 1e-30)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def assert_bf16_close(gpu: np.ndarray, ref: np.ndarray, name: str, max_abs=MAX_ABS,
                      rel_rms=REL_RMS) -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{name}: non-finite output"
    err = np.abs(gpu - ref)
    tol = np.where(np.abs(ref) < 8.0, max_abs, max_abs + half_ulp_bf16(ref))
    worst = int(np.argmax(err - tol))
    rr = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30))
    stats = dict(name=name, max_abs=float(err.max()) if err.size else 0.0, rel_rms=rr,
                 n_ge8=int((np.abs(ref) >= 8).sum()))
    assert (err <= tol).all(), (f"{name}: max-abs {err.flat[worst]:.4g} > {tol.flat[worst]:.4g} "
                                f"at {np.unravel_index(worst, err.shape)}; {stats}")
    assert rr <= rel_rms, f"{name}: relative RMS {rr:.3g} > {rel_rms}; {stats}"
    return stats


class DevicePack:
    """A workload's inputs and pack metadata in device memory, built by the
    library's own mf_pack_build / mf_adaln_params."""

    def __init__(self, w: Workload, stream=None):
        self.w = w
        self.S, self.H, self.D, self.hid = w.S, w.H, w.D, w.hid
        self.cu_h, self.T = mf.mf_pack_build(w.descs, w.rope_axes, w.budget)
        T = self.T
        self.cu_d = torch.empty(w.S + 1, dtype=torch.int32, device="cuda")
        self.pos = torch.empty((max(T, 1), 3), dtype=torch.int32, device="cuda")
        self.tok_sample = torch.empty(max(T, 1), dtype=torch.int32, device="cuda")
        self.tok_mod = torch.empty(max(T, 1), dtype=torch.uint8, device="cuda")
        mf.mf_pack_build(w.descs, w.rope_axes, w.budget, self.cu_d, self.pos, self.tok_sample,
                         self.tok_mod)
        self.x = dev_bf16(w.x_bits.reshape(T, w.hid)) if T else None
        self.q = dev_bf16(w.q_bits) if T else None
        self.k = dev_bf16(w.k_bits) if T else None
        self.v = dev_bf16(w.v_bits) if T else None
        self.c = torch.from_numpy(w.c).cuda()
        self.W = torch.from_numpy(w.W).cuda()
        self.mod = torch.empty((w.S, 2, 3, w.hid), dtype=torch.float32, device="cuda")
        mf.mf_adaln_params(self.c, self.W, w.S, self.c.shape[1], w.hid, self.mod)
        self.ws_bytes = mf.mf_workspace_size(T, w.H, w.D, 1)
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device="cuda")

    def block(self):
        T, hid = self.T, self.hid
        x_mod = torch.empty((T, hid), dtype=torch.bfloat16, device="cuda")
        y = torch.empty((T, hid), dtype=torch.bfloat16, device="cuda")
        mf.mf_block_fwd(self.x, self.q, self.k, self.v, self.mod, self.cu_d, self.cu_h, self.pos,
                        self.tok_sample, self.tok_mod, self.S, self.H, self.D, self.w.rope_axes,
                        self.w.base, self.w.eps, x_mod, y, self.ws, self.ws_bytes)
        return x_mod, y

    def attention(self, q, k, v, with_rope: bool, lse: bool = False):
        T = self.T
        o = torch.empty((T, self.H, self.D), dtype=torch.bfloat16, device="cuda")
        lse_t = torch.empty((self.H, T), dtype=torch.float32, device="cuda") if lse else None
        mf.mf_varlen_attn_fwd(q, k, v, self.cu_d, self.cu_h, self.S, self.H, self.D,
                              1.0 / math.sqrt(self.D), self.pos if with_rope else None,
                              self.w.rope_axes, self.w.base, o, lse_t, self.ws if with_rope else None,
                              self.ws_bytes if with_rope else 0)
        return o, lse_t


def sample_rows(cu: np.ndarray, per_sample: int, seed: int) -> np.ndarray:
    """Query rows to check at full size: both ends of every sample, the rows
    around each 128-row tile boundary, and random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        if hi <= lo:
            continue
        rows.update([lo, hi - 1])
        for b in range(lo + 127, hi, 128 * max(1, (hi - lo) // (128 * 8))):
            rows.update(r for r in (b, b + 1) if lo <= r < hi)
        rows.update(int(r) for r in rng.integers(lo, hi, size=min(per_sample, hi - lo)))
    return np.array(sorted(rows), dtype=np.int64)


def oracle_pack(w: Workload):
    return oracle.pack_build(w.descs, w.rope_axes)


def zero_grad_bound(q, k, v, d_o, D: int) -> float:
    """A one-token sample has P = 1, so dS = dP - rowsum(dO * O) = dO.v - dO.v is
    exactly 0 and so are its dQ and dK. The kernel forms the two dot products in
    fp32 in different orders (tensor-core dP against the row table's delta, from
    O = v stored in bf16, which is exact), so their difference is bounded by the
    fp32 summation bound of two D-term sums, 2 * D * 2^-24 * sum|dO v|; dQ and dK
    are that times scale * max|k| (resp. |q|)."""
    terms = np.abs(d_o.astype(np.float64) * v.astype(np.float64)).sum(axis=-1).max()
    big = max(np.abs(q).max(), np.abs(k).max())
    return float(2 * D * 2.0 ** -24 * terms / math.sqrt(D) * big)


def assert_grad_close(gpu: np.ndarray, ref: np.ndarray, cu, name: str, zero_tol=0.0) -> list:
    """Per sample: relative RMS <= GRAD_REL_RMS and max error <= GRAD_MAX_REL * max|ref|;
    for dQ and dK (zero_tol > 0) a one-token sample, whose exact gradient is 0
    (see zero_grad_bound), must stay within zero_tol."""
    stats = []
    assert np.isfinite(gpu).all(), f"{name}: non-finite gradient"
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        if hi == lo:
            continue
        g, r = gpu[lo:hi].astype(np.float64), ref[lo:hi]
        if hi - lo == 1 and zero_tol > 0:  # dQ, dK of a one-token sample: exactly 0
            worst = float(np.abs(g).max())
            stats.append((name, s, hi - lo, 0.0, worst))
            assert worst <= zero_tol, f"{name} sample {s}: exact zero, got {worst:.3g} > {zero_tol:.3g}"
            continue
        scale = float(np.abs(r).max())
        err = np.abs(g - r)
        rr = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))
        mr = float(err.max() / max(scale, 1e-300))
        stats.append((name, s, hi - lo, rr, mr))
        assert rr <= GRAD_REL_RMS, f"{name} sample {s}: relative RMS {rr:.3g} > {GRAD_REL_RMS}"
        assert mr <= GRAD_MAX_REL, f"{name} sample {s}: max error {mr:.3g} of max|ref| > {GRAD_MAX_REL}"
    return stats


def assert_block_close(got, ref, name):
    """For a chain whose output adds bf16-stored intermediates (the MMDiT
    block's y1, the VAE block's activations) that the GPU and the oracle round
    independently, from fp32 and fp64 values: one bf16 ulp of such an
    intermediate can separate them on top of the output's own rounding. The
    bound is therefore max-abs 2e-2 plus one bf16 ulp at the value's
    magnitude, with the relative RMS bound unchanged (5e-3)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape and np.isfinite(got).all(), name
    err = np.abs(got - ref)
    tol = MAX_ABS + 2.0 * half_ulp_bf16(ref)
    worst = int(np.argmax(err - tol))
    assert (err <= tol).all(), (f"{name}: |err| {err.flat[worst]:.4g} > {tol.flat[worst]:.4g} at "
                                f"{np.unravel_index(worst, err.shape)}")
    rr = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert rr <= REL_RMS, f"{name}: relative RMS {rr:.3g}"
