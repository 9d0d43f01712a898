"""The C-ABI library without a GPU: it loads, exports every symbol include/mf.h
declares, and its host-side logic (pack offsets, argument checks, workspace
sizing) matches the oracle and the header's contract. No compute is launched."""

import ctypes

import numpy as np
import pytest

import oracle
from packgen import SampleDesc, make_random_pack, make_workload

mf = pytest.importorskip("resolution_packed_diffusion_b200")


def test_library_exports_every_declared_symbol():
    names = mf.header_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(mf.lib, n), n
        assert n in mf._SIGS, f"binding lacks {n}"
    for needed in ("mf_pack_build", "mf_adaln_modulate", "mf_rope_apply", "mf_varlen_attn_fwd",
                   "mf_gated_residual", "mf_block_fwd"):
        assert needed in names


def test_abi_version_and_status_strings():
    assert mf.abi_version() == 1
    assert mf.status_string(mf.MF_OK) == "MF_OK"
    assert mf.status_string(mf.MF_ERR_TIMEOUT) == "MF_ERR_TIMEOUT"


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_pack_offsets_match_oracle(idx):
    w = make_workload(idx, with_arrays=False)
    cu, T = mf.mf_pack_build(w.descs, w.rope_axes, w.budget)
    ref = oracle.pack_build(w.descs, w.rope_axes)
    assert T == ref["T"] == w.T
    assert np.array_equal(cu, ref["cu_seqlens"])


def test_pack_offsets_random_and_empty():
    for seed in range(20):
        axes = 2 + seed % 2
        w = make_random_pack(seed, S=1 + seed % 7, H=1, D=8, rope_axes=axes, max_grid=9,
                             max_text=11)
        cu, T = mf.mf_pack_build(w.descs, axes, 0)
        assert np.array_equal(cu, oracle.pack_build(w.descs, axes)["cu_seqlens"])
    cu, T = mf.mf_pack_build([], 2, 0)
    assert T == 0 and cu.tolist() == [0]


@pytest.mark.parametrize("descs,axes,budget", [
    ([(2, 4, 4, 3)], 2, 0),           # two frames need the 3D layout
    ([(3, 4, 4, 3)], 3, 0),           # at most two frames
    ([(1, -1, 4, 3)], 2, 0),          # negative grid
    ([(1, 4, 4, -2)], 2, 0),          # negative text length
    ([(1, 64, 64, 256)], 2, 1000),    # over the token budget
    ([(1, 4, 4, 0)], 4, 0),           # bad rope_axes
])
def test_pack_rejects_invalid(descs, axes, budget):
    with pytest.raises(mf.MFError) as e:
        mf.mf_pack_build(descs, axes, budget)
    assert e.value.status == mf.MF_ERR_INVALID


def test_pack_rejects_too_many_samples():
    with pytest.raises(mf.MFError):
        mf.mf_pack_build([(1, 1, 1, 1)] * (mf.MF_MAX_SAMPLES + 1), 2, 0)


def test_workspace_size():
    """The fused RoPE's workspace: its (cos, sin) table, T positions x D/4 pair
    columns of two floats (the 2D split has D/4 pairs per axis, the 3D one
    fewer), and the rotated k, T x H x D bf16."""
    assert mf.mf_workspace_size(0, 24, 128, 1) == 0
    assert mf.mf_workspace_size(100, 24, 128, 0) == 0
    for D in (64, 128):
        need = 100 * (D // 4) * 8 + 100 * 24 * D * 2
        assert need <= mf.mf_workspace_size(100, 24, D, 1) <= need + 768


def test_host_argument_checks_without_gpu():
    """Calls that fail validation return before touching the GPU."""
    lib = mf.lib
    cu = np.array([0, 10], dtype=np.int32)
    P = ctypes.c_void_p
    # head_dim 96 is outside the supported set
    st = lib.mf_varlen_attn_fwd(P(16), P(16), P(16), P(16), cu.ctypes.data_as(P), 1, 2, 96,
                                0.1, None, 2, 10000.0, P(4096), None, None, 0, None)
    assert st == mf.MF_ERR_UNSUPPORTED
    # misaligned output pointer
    st = lib.mf_varlen_attn_fwd(P(16), P(16 + 4096), P(16 + 8192), P(16), cu.ctypes.data_as(P),
                                1, 1, 64, 0.1, None, 2, 10000.0, P(1 << 20 | 8), None, None, 0,
                                None)
    assert st == mf.MF_ERR_INVALID
    # non-monotone offsets
    bad = np.array([0, 10, 5], dtype=np.int32)
    st = lib.mf_varlen_attn_fwd(P(16), P(16), P(16), P(16), bad.ctypes.data_as(P), 2, 1, 64,
                                0.1, None, 2, 10000.0, P(4096), None, None, 0, None)
    assert st == mf.MF_ERR_INVALID
    # non-positive softmax scale
    st = lib.mf_varlen_attn_fwd(P(16), P(1 << 20), P(2 << 20), P(16), cu.ctypes.data_as(P), 1,
                                1, 64, 0.0, None, 2, 10000.0, P(4 << 20), None, None, 0, None)
    assert st == mf.MF_ERR_INVALID
    # empty pack: nothing to do
    z = np.array([0, 0], dtype=np.int32)
    st = lib.mf_varlen_attn_fwd(None, None, None, None, z.ctypes.data_as(P), 1, 1, 64, 0.1,
                                None, 2, 10000.0, None, None, None, 0, None)
    assert st == mf.MF_OK
    # adaLN: hid above the supported row length
    st = lib.mf_adaln_modulate(P(16), P(16), P(16), P(16), 4, 1, 8192, 1e-6, P(1 << 30), None)
    assert st == mf.MF_ERR_UNSUPPORTED
    # RoPE with no tensor to rotate
    st = lib.mf_rope_apply(None, None, P(16), 4, 1, 64, 2, 10000.0, None, None, None)
    assert st == mf.MF_ERR_INVALID
    # block forward with too small a workspace
    cu2 = np.array([0, 128], dtype=np.int32)
    st = lib.mf_block_fwd(P(1 << 24), P(2 << 24), P(3 << 24), P(4 << 24), P(5 << 24), P(16),
                          cu2.ctypes.data_as(P), P(16), P(16), P(16), 1, 2, 64, 2, 10000.0,
                          1e-6, P(6 << 24), P(7 << 24), P(8 << 24), 16, None)
    assert st == mf.MF_ERR_INVALID


def test_cfg_combine_argument_checks_launch_nothing():
    """Invalid pairs, widths or weights are refused on the host (no GPU is
    touched: the checks come before any launch)."""
    descs = mf.make_descs([(1, 3, 4, 5), (0, 0, 0, 7), (1, 3, 4, 2), (1, 2, 2, 1)])
    fake = 1 << 20  # 16-byte aligned stand-in pointers, never dereferenced

    def call(pairs, C=8, w=1.0, S=4):
        parr = (mf.mf_cfg_pair * max(1, len(pairs)))(*[mf.mf_cfg_pair(c, u) for c, u in pairs])
        return mf.lib.mf_cfg_combine(fake, ctypes.cast(descs, ctypes.c_void_p), S,
                                     ctypes.cast(parr, ctypes.c_void_p), len(pairs), C, w,
                                     fake + (1 << 30), None)
    assert call([(0, 3)]) == mf.MF_ERR_INVALID      # 12 vs 4 image tokens
    assert call([(2, 2)]) == mf.MF_ERR_INVALID      # a sample paired with itself
    assert call([(0, 4)]) == mf.MF_ERR_INVALID      # out of range
    assert call([(0, 2)], C=12) == mf.MF_ERR_INVALID
    assert call([(0, 2)], w=float("inf")) == mf.MF_ERR_INVALID
    assert call([]) == mf.MF_ERR_INVALID            # no pairs


def test_backward_argument_checks_without_gpu():
    """The backward entry points validate before touching the GPU."""
    lib = mf.lib
    P = ctypes.c_void_p
    cu = np.array([0, 10], dtype=np.int32)
    T, H, D = 10, 2, 64
    ws = mf.mf_attn_bwd_workspace_size(T, 1, H, D)
    assert ws >= T * H * D * 4
    assert mf.mf_attn_bwd_workspace_size(2 * T, 1, H, D) > ws
    MB = 1 << 20
    q, k, v, o, do, lse = (P((i + 1) * MB) for i in range(6))
    dq, dk, dv, w = (P((i + 10) * MB) for i in range(4))

    def call(D=D, scale=0.125, dq=dq, dk=dk, dv=dv, w=w, ws=ws, cu=cu):
        return lib.mf_varlen_attn_bwd(q, k, v, o, do, lse, P(16), cu.ctypes.data_as(P),
                                      len(cu) - 1, H, D, scale, dq, dk, dv, w, ws, None)

    assert call(D=96) == mf.MF_ERR_UNSUPPORTED
    assert call(scale=0.0) == mf.MF_ERR_INVALID
    assert call(dq=q) == mf.MF_ERR_INVALID            # an output aliases an input
    assert call(dv=dk) == mf.MF_ERR_INVALID           # two outputs share a buffer
    assert call(w=dq) == mf.MF_ERR_INVALID            # workspace overlaps an output
    assert call(ws=ws - 256) == mf.MF_ERR_INVALID     # workspace too small
    assert call(dq=P(10 * MB + 8)) == mf.MF_ERR_INVALID  # misaligned
    assert call(cu=np.array([0, 10, 5], dtype=np.int32)) == mf.MF_ERR_INVALID
    assert call(cu=np.array([0, 0], dtype=np.int32)) == mf.MF_OK  # empty pack: nothing to do
    # RoPE backward: same checks as the forward rotation
    assert lib.mf_rope_bwd(None, None, P(16), 4, 1, 64, 2, 10000.0, None, None, None) == \
        mf.MF_ERR_INVALID
    assert lib.mf_rope_bwd(q, None, P(16), 4, 1, 64, 4, 10000.0, dq, None, None) == \
        mf.MF_ERR_INVALID
    assert lib.mf_rope_bwd(q, None, P(16), 4, 1, 96, 2, 10000.0, dq, None, None) == \
        mf.MF_ERR_UNSUPPORTED


def test_gate_and_adaln_backward_argument_checks_without_gpu():
    lib = mf.lib
    P = ctypes.c_void_p
    MB = 1 << 20
    T, S, hid = 100, 2, 64
    dy, o, mod, ts, tm, d_o, dmod = (P((i + 1) * MB) for i in range(7))
    assert lib.mf_gated_residual_bwd(dy, o, mod, ts, tm, T, S, 60, d_o, dmod, None) == \
        mf.MF_ERR_INVALID                                        # hid not a multiple of 8
    assert lib.mf_gated_residual_bwd(dy, o, mod, ts, tm, T, S, hid, o, dmod, None) == \
        mf.MF_ERR_INVALID                                        # d_o overlaps o
    assert lib.mf_gated_residual_bwd(dy, o, mod, ts, tm, T, S, hid, d_o, mod, None) == \
        mf.MF_ERR_INVALID                                        # dmod overlaps mod
    assert lib.mf_gated_residual_bwd(dy, o, mod, ts, tm, T, 0, hid, d_o, dmod, None) == \
        mf.MF_ERR_INVALID                                        # no samples
    ws = mf.mf_adaln_bwd_workspace_size(T)
    assert ws >= T * 8 and mf.mf_adaln_bwd_workspace_size(0) == 0
    x, dxm, dx, w = P(20 * MB), P(21 * MB), P(22 * MB), P(23 * MB)

    def ln(dx=dx, resid=None, eps=1e-6, w=w, ws=ws):
        return lib.mf_adaln_modulate_bwd(dxm, x, mod, ts, tm, resid, T, S, hid, eps, dx, dmod, w,
                                         ws, None)

    assert ln(eps=0.0) == mf.MF_ERR_INVALID
    assert ln(dx=x) == mf.MF_ERR_INVALID                         # dx overlaps x
    assert ln(dx=dxm) == mf.MF_ERR_INVALID                       # dx overlaps dx_mod
    assert ln(ws=ws - 1) == mf.MF_ERR_INVALID                    # workspace too small
    assert ln(w=dx) == mf.MF_ERR_INVALID                         # workspace overlaps dx
    assert ln(resid=P(22 * MB + 64)) == mf.MF_ERR_INVALID        # partial overlap with resid

    assert lib.mf_gated_residual_bwd(dy, o, mod, ts, tm, T, S, hid, d_o, dy, None) == \
        mf.MF_ERR_INVALID                                        # dmod overlaps dy
    assert lib.mf_gated_residual_bwd(dy, o, mod, ts, tm, T, S, hid, mod, dmod, None) == \
        mf.MF_ERR_INVALID                                        # d_o overlaps mod
    assert ln(w=x) == mf.MF_ERR_INVALID                          # workspace overlaps x
    assert lib.mf_adaln_modulate_bwd(dxm, x, mod, ts, tm, None, T, S, hid, 1e-6, dx, x, w, ws,
                                     None) == mf.MF_ERR_INVALID  # dmod overlaps x


def test_forward_workspace_and_output_overlap_checks_without_gpu():
    """The forward entry points refuse a workspace that overlaps an input or an
    output, and outputs that overlap the modulation vectors: the rotated Q and K
    are written while other CTAs still read q and k, and the fused epilogue
    reads x, v and mod while y is written."""
    lib = mf.lib
    P = ctypes.c_void_p
    MB = 1 << 20
    T, H, D = 128, 2, 64
    cu = np.array([0, T], dtype=np.int32)
    x, q, k, v, mod, xm, y, ws, pos = (P((i + 1) * MB) for i in range(9))
    wsb = mf.mf_workspace_size(T, H, D, 1)

    def blk(ws=ws, xm=xm, y=y, mod=mod, pos=pos):
        return lib.mf_block_fwd(x, q, k, v, mod, P(16), cu.ctypes.data_as(P), pos, P(16), P(16),
                                1, H, D, 2, 10000.0, 1e-6, xm, y, ws, wsb, None)

    for bad in (x, q, k, v, mod, xm, y, pos):
        assert blk(ws=bad) == mf.MF_ERR_INVALID
    assert blk(ws=P(q.value + 4096)) == mf.MF_ERR_INVALID   # partial overlap
    assert blk(xm=mod) == mf.MF_ERR_INVALID
    assert blk(y=P(mod.value + 256)) == mf.MF_ERR_INVALID

    def attn(ws=ws, o=y, lse=None):
        return lib.mf_varlen_attn_fwd(q, k, v, P(16), cu.ctypes.data_as(P), 1, H, D, 0.125, pos,
                                      2, 10000.0, o, lse, ws, wsb, None)

    for bad in (q, k, v, y, pos):
        assert attn(ws=bad) == mf.MF_ERR_INVALID
    assert attn(lse=ws) == mf.MF_ERR_INVALID


@pytest.mark.parametrize("offsets", [[5, 100], [0, 50000, 40000, 9000000],
                                     [0, (1 << 24) + 64]])
def test_noalloc_rejects_malformed_offsets_as_invalid(offsets):
    """A malformed pack is an argument error whatever its last offset (the size
    test against the fixed array comes after the offsets are validated)."""
    P = ctypes.c_void_p
    cu = np.array(offsets, dtype=np.int32)
    st = mf.lib.mf_block_fwd_noalloc(P(16), P(16), P(16), P(16), P(16), P(16),
                                     cu.ctypes.data_as(P), P(16), P(16), P(16), len(cu) - 1, 24,
                                     128, 2, 10000.0, 1e-6, P(16), P(16), None)
    assert st == mf.MF_ERR_INVALID


def test_noalloc_size_limit_without_gpu():
    P = ctypes.c_void_p
    cu = np.array([0, 16384], dtype=np.int32)  # 16384 x 3072 rotated k plus table: ~105 MB
    st = mf.lib.mf_block_fwd_noalloc(P(16), P(16), P(16), P(16), P(16), P(16),
                                     cu.ctypes.data_as(P), P(16), P(16), P(16), 1, 24, 128, 2,
                                     10000.0, 1e-6, P(16), P(16), None)
    assert st == mf.MF_ERR_UNSUPPORTED


def test_adaln_params_bwd_argument_checks_without_gpu():
    lib = mf.lib
    P = ctypes.c_void_p
    MB = 1 << 20
    dmod, c, W, dc, dW = (P((i + 1) * 16 * MB) for i in range(5))

    def call(dc=dc, dW=dW, S=3, C=128, hid=3072):
        return lib.mf_adaln_params_bwd(dmod, c, W, S, C, hid, dc, dW, None)

    assert call(dc=None, dW=None) == mf.MF_ERR_INVALID           # nothing to compute
    assert call(hid=3076) == mf.MF_ERR_INVALID                   # hid not a multiple of 8
    assert call(S=0) == mf.MF_ERR_INVALID
    assert call(dc=W) == mf.MF_ERR_INVALID                       # dc overlaps W
    assert call(dW=P(dmod.value + 64)) == mf.MF_ERR_INVALID      # dW overlaps dmod
    assert call(dW=P(dc.value)) == mf.MF_ERR_INVALID             # the outputs overlap
    assert call(dc=P(dc.value + 8)) == mf.MF_ERR_INVALID         # misaligned


def test_vae_argument_checks_without_gpu():
    """The VAE entry points validate shapes, alignment and overlaps before
    touching the GPU; workspace sizes follow the documented layout."""
    lib = mf.lib
    P = ctypes.c_void_p
    MB = 1 << 20
    x, Wt, y, b, ws = (P((i + 1) * 64 * MB) for i in range(5))
    assert lib.mf_conv3x3(x, Wt, None, None, 1, 8, 8, 96, 64, y, None) == mf.MF_ERR_UNSUPPORTED
    assert lib.mf_conv3x3(x, Wt, None, None, 1, 8, 8, 64, 4096, y, None) == mf.MF_ERR_UNSUPPORTED
    assert lib.mf_conv3x3(x, Wt, None, None, 0, 8, 8, 64, 64, y, None) == mf.MF_ERR_INVALID
    assert lib.mf_conv3x3(x, Wt, None, None, 1, 8, 8, 64, 64, x, None) == mf.MF_ERR_INVALID
    assert lib.mf_conv3x3(x, Wt, None, P(y.value + 256), 1, 8, 8, 64, 64, y, None) == \
        mf.MF_ERR_INVALID                                      # residual partly over y
    assert lib.mf_conv3x3(x, Wt, P(b.value + 4), None, 1, 8, 8, 64, 64, y, None) == \
        mf.MF_ERR_INVALID                                      # misaligned bias
    gws = mf.mf_gn_workspace_size(1, 8, 8, 8)
    assert gws > 0 and mf.mf_gn_workspace_size(0, 8, 8, 8) == 0

    def gn(C=64, G=8, y=y, ws=ws, wsb=gws, eps=1e-6):
        return lib.mf_group_norm_silu(x, b, b, 1, 8, 8, C, G, eps, y, ws, wsb, None)

    assert gn(G=16) == mf.MF_ERR_UNSUPPORTED                   # 4 channels a group
    assert gn(C=96, G=12) == mf.MF_ERR_UNSUPPORTED
    assert gn(y=x) == mf.MF_ERR_INVALID
    assert gn(wsb=gws - 1) == mf.MF_ERR_INVALID
    assert gn(ws=x) == mf.MF_ERR_INVALID
    assert gn(eps=float("nan")) == mf.MF_ERR_INVALID
    act = 1 * 8 * 8 * 64 * 2
    assert mf.mf_vae_block_workspace_size(1, 8, 8, 64, 8) >= 2 * act + gws
    assert lib.mf_vae_res_block(x, b, b, Wt, b, b, b, Wt, b, 1, 8, 8, 64, 8, 1e-6, y, x,
                                mf.mf_vae_block_workspace_size(1, 8, 8, 64, 8), None) == \
        mf.MF_ERR_INVALID                                      # workspace over x


def test_mmdit_block_bwd_argument_checks_without_gpu():
    """The block backward checks shapes, the descriptors against the offsets,
    alignment, workspace size and overlaps before touching the GPU."""
    lib = mf.lib
    P = ctypes.c_void_p
    MB = 1 << 20
    descs = [SampleDesc(1, 4, 4, 3), SampleDesc(0, 0, 0, 5)]
    arr = mf.make_descs(descs)
    cu = np.array([0, 19, 24], dtype=np.int32)
    S, H, D, F = 2, 2, 128, 512
    T = 24
    ws_size = mf.mf_mmdit_bwd_workspace_size(T, S, H, D, F)
    assert ws_size > 0 and mf.mf_mmdit_bwd_workspace_size(T, 0, H, D, F) == 0
    ptr = [P((i + 1) * 64 * MB) for i in range(22)]
    (dy, x, Wq, Wk, Wv, Wo, Wup, Wdown, ma, mm, dx, dWq, dWk, dWv, dWo, dWup, dWdown, dma, dmm,
     ws, pos, ids) = ptr

    def call(H=H, D=D, F=F, cu=cu, dx=dx, dWq=dWq, ws=ws, ws_bytes=ws_size):
        return lib.mf_mmdit_block_bwd(dy, x, Wq, Wk, Wv, Wo, Wup, Wdown, ma, mm,
                                      ctypes.cast(arr, P), P(16), cu.ctypes.data_as(P), pos, ids,
                                      ids, S, H, D, F, 2, 10000.0, 1e-6, dx, dWq, dWk, dWv, dWo,
                                      dWup, dWdown, dma, dmm, ws, ws_bytes, None)

    assert call(F=500) == mf.MF_ERR_INVALID                         # F not a multiple of 256
    assert call(F=131072 + 256) == mf.MF_ERR_UNSUPPORTED            # beyond the job table
    assert call(D=64) == mf.MF_ERR_UNSUPPORTED                      # hid 128
    assert call(cu=np.array([0, 18, 24], dtype=np.int32)) == mf.MF_ERR_INVALID  # desc vs offsets
    assert call(cu=np.array([0, 19, 18], dtype=np.int32)) == mf.MF_ERR_INVALID  # decreasing
    assert call(dx=x) == mf.MF_ERR_INVALID                          # output over an input
    assert call(dWq=P(dWk.value + 64)) == mf.MF_ERR_INVALID         # two outputs overlap
    assert call(dWq=P(dWq.value + 8)) == mf.MF_ERR_INVALID          # misaligned
    assert call(ws_bytes=ws_size - 1) == mf.MF_ERR_INVALID
    assert call(ws=P(dx.value + 256)) == mf.MF_ERR_INVALID          # workspace over dx
