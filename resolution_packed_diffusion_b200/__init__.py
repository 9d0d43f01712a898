"""Python binding of libmf, the sm_100a packed joint-attention block.

Argument marshalling only: every function here has the name and argument order
of the C entry point in ``include/mf.h``; tensors stand in for pointers (their
``data_ptr()`` is passed), ``None`` for NULL, and the current torch CUDA stream
is used unless ``stream`` is given. Every step of the block runs in libmf's
CUDA kernels. There is no CPU fallback: importing this package fails loudly if
``libmf.so`` has not been built (``python resolution_packed_diffusion_b200/build.py``).
"""

from __future__ import annotations

import ctypes
import os
import re
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmf.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "mf.h")

MF_OK, MF_ERR_INVALID, MF_ERR_CUDA, MF_ERR_TIMEOUT, MF_ERR_UNSUPPORTED = 0, 1, 2, 3, 4
MF_MAX_SAMPLES = 512
MF_NOALLOC_SCRATCH_BYTES = 64 << 20


class MFError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == MF_ERR_CUDA:
            detail = " (" + lib.mf_last_error_detail().decode() + ")"
        super().__init__(f"{where}: {status_string(status)}{detail}")


class mf_sample_desc(ctypes.Structure):
    _fields_ = [("frames", ctypes.c_int32), ("grid_h", ctypes.c_int32),
                ("grid_w", ctypes.c_int32), ("n_text", ctypes.c_int32),
                ("is_dummy", ctypes.c_int32)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python resolution_packed_diffusion_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_U64 = ctypes.c_uint64

_SIGS = {
    "mf_abi_version": (_I, []),
    "mf_status_string": (ctypes.c_char_p, [_I]),
    "mf_last_error_detail": (ctypes.c_char_p, []),
    "mf_pack_build": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "mf_adaln_params": (_I, [_P, _P, _I, _I, _I, _P, _P]),
    "mf_adaln_modulate": (_I, [_P, _P, _P, _P, _I, _I, _I, _F, _P, _P]),
    "mf_adaln_params_bwd": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "mf_rope_apply": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _P, _P]),
    "mf_rope_bwd": (_I, [_P, _P, _P, _I, _I, _I, _I, _F, _P, _P, _P]),
    "mf_varlen_attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _F, _P, _I, _F, _P, _P, _P,
                                _SZ, _P]),
    "mf_varlen_attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _F, _P, _P, _P, _P,
                                _SZ, _P]),
    "mf_attn_bwd_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "mf_gated_residual": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "mf_gated_residual_bwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "mf_adaln_modulate_bwd": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _F, _P, _P, _P, _SZ,
                                   _P]),
    "mf_adaln_bwd_workspace_size": (_SZ, [_I]),
    "mf_block_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _F, _P,
                          _P, _P, _SZ, _P]),
    "mf_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "mf_get_error": (_I, [_P]),
    "mf_set_wait_limit_ns": (_I, [_U64]),
    "mf_selftest_wait_timeout": (_I, [_U64, _P]),
    "mf_selftest_exp2_poly": (_I, [_P, _P, _I, _P]),
    "mf_set_attn_timing_events": (_I, [_P, _P]),
    "mf_set_attn_cta_pair": (_I, [_I]),
    "mf_set_linear_cta_pair": (_I, [_I]),
    "mf_set_conv_cta_pair": (_I, [_I]),
    "mf_block_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F,
                                  _F, _P, _P, _P]),
    "mf_cfg_combine": (_I, [_P, _P, _I, _P, _I, _I, _F, _P, _P]),
    "mf_modality_linear": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "mf_mmdit_block_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I,
                                _I, _I, _I, _I, _F, _F, _P, _P, _SZ, _P]),
    "mf_mmdit_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "mf_mmdit_block_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                _I, _I, _I, _I, _I, _F, _F, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                _P, _SZ, _P]),
    "mf_mmdit_bwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "mf_group_norm_silu": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P, _SZ, _P]),
    "mf_gn_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "mf_conv3x3": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "mf_vae_res_block": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P,
                              _SZ, _P]),
    "mf_vae_block_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def header_symbols(path: str = HEADER_PATH) -> List[str]:
    """Names of the functions ``include/mf.h`` declares."""
    text = open(path).read()
    return sorted(set(re.findall(r"^(?:const\s+)?\w+\s*\*?\s*(mf_\w+)\(", text, re.M)))


def status_string(status: int) -> str:
    return lib.mf_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MF_OK:
        raise MFError(status, where)


def _ptr(t) -> Optional[int]:
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libmf entry points take device tensors")
    if not t.is_contiguous():
        raise ValueError("libmf entry points take contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_descs(descs: Iterable) -> ctypes.Array:
    """ctypes array of mf_sample_desc from (frames, grid_h, grid_w, n_text[, is_dummy])
    tuples or objects with ``as_tuple()``."""
    rows = [tuple(d.as_tuple()) if hasattr(d, "as_tuple") else tuple(d) for d in descs]
    arr = (mf_sample_desc * max(1, len(rows)))()
    for i, r in enumerate(rows):
        r = tuple(r) + (0,) * (5 - len(r))
        arr[i] = mf_sample_desc(*[int(v) for v in r[:5]])
    return arr


def abi_version() -> int:
    return lib.mf_abi_version()


def mf_pack_build(descs, rope_axes: int, budget: int = 0, cu_seqlens_d=None, pos_ids_d=None,
                  tok_sample_d=None, tok_mod_d=None, stream=None) -> Tuple[np.ndarray, int]:
    """Returns (cu_seqlens_h as int32 [S+1], T). With all device tensors None
    this is a host-only size query."""
    arr = make_descs(descs)
    S = len(list(descs)) if not isinstance(descs, ctypes.Array) else len(descs)
    cu_h = np.zeros(S + 1, dtype=np.int32)
    T = ctypes.c_int32(0)
    query = all(t is None for t in (cu_seqlens_d, pos_ids_d, tok_sample_d, tok_mod_d))
    st = None if query else _stream(stream)
    _check(lib.mf_pack_build(ctypes.cast(arr, _P), S, rope_axes, budget,
                             cu_h.ctypes.data_as(_P), _ptr(cu_seqlens_d), _ptr(pos_ids_d),
                             _ptr(tok_sample_d), _ptr(tok_mod_d), ctypes.byref(T), st),
           "mf_pack_build")
    return cu_h, int(T.value)


def mf_adaln_params(c, W, S: int, C: int, hid: int, mod, stream=None) -> None:
    _check(lib.mf_adaln_params(_ptr(c), _ptr(W), S, C, hid, _ptr(mod), _stream(stream)),
           "mf_adaln_params")


def mf_adaln_params_bwd(dmod, c, W, S: int, C: int, hid: int, dc, dW, stream=None) -> None:
    _check(lib.mf_adaln_params_bwd(_ptr(dmod), _ptr(c), _ptr(W), S, C, hid, _ptr(dc), _ptr(dW),
                                   _stream(stream)), "mf_adaln_params_bwd")


def mf_adaln_modulate(x, mod, tok_sample, tok_mod, T: int, S: int, hid: int, eps: float, x_mod,
                      stream=None) -> None:
    _check(lib.mf_adaln_modulate(_ptr(x), _ptr(mod), _ptr(tok_sample), _ptr(tok_mod), T, S, hid,
                                 eps, _ptr(x_mod), _stream(stream)), "mf_adaln_modulate")


def mf_rope_apply(q, k, pos_ids, T: int, H: int, D: int, rope_axes: int, base: float, q_out,
                  k_out, stream=None) -> None:
    _check(lib.mf_rope_apply(_ptr(q), _ptr(k), _ptr(pos_ids), T, H, D, rope_axes, base,
                             _ptr(q_out), _ptr(k_out), _stream(stream)), "mf_rope_apply")


def mf_rope_bwd(dq_r, dk_r, pos_ids, T: int, H: int, D: int, rope_axes: int, base: float, dq,
                dk, stream=None) -> None:
    _check(lib.mf_rope_bwd(_ptr(dq_r), _ptr(dk_r), _ptr(pos_ids), T, H, D, rope_axes, base,
                           _ptr(dq), _ptr(dk), _stream(stream)), "mf_rope_bwd")


def mf_varlen_attn_fwd(q, k, v, cu_seqlens_d, cu_seqlens_h: np.ndarray, S: int, H: int, D: int,
                       softmax_scale: float, pos_ids, rope_axes: int, base: float, o, lse,
                       workspace, ws_bytes: int, stream=None) -> None:
    cu_h = np.ascontiguousarray(cu_seqlens_h, dtype=np.int32)
    _check(lib.mf_varlen_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_d),
                                  cu_h.ctypes.data_as(_P), S, H, D, softmax_scale,
                                  _ptr(pos_ids), rope_axes, base, _ptr(o), _ptr(lse),
                                  _ptr(workspace), ws_bytes, _stream(stream)),
           "mf_varlen_attn_fwd")


def mf_varlen_attn_bwd(q, k, v, o, d_o, lse, cu_seqlens_d, cu_seqlens_h: np.ndarray, S: int,
                       H: int, D: int, softmax_scale: float, dq, dk, dv, workspace,
                       ws_bytes: int, stream=None) -> None:
    cu_h = np.ascontiguousarray(cu_seqlens_h, dtype=np.int32)
    _check(lib.mf_varlen_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(d_o), _ptr(lse),
                                  _ptr(cu_seqlens_d), cu_h.ctypes.data_as(_P), S, H, D,
                                  softmax_scale, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                  ws_bytes, _stream(stream)),
           "mf_varlen_attn_bwd")


def mf_attn_bwd_workspace_size(T: int, S: int, H: int, D: int) -> int:
    return int(lib.mf_attn_bwd_workspace_size(T, S, H, D))


def mf_gated_residual_bwd(dy, o, mod, tok_sample, tok_mod, T: int, S: int, hid: int, d_o, dmod,
                          stream=None) -> None:
    _check(lib.mf_gated_residual_bwd(_ptr(dy), _ptr(o), _ptr(mod), _ptr(tok_sample),
                                     _ptr(tok_mod), T, S, hid, _ptr(d_o), _ptr(dmod),
                                     _stream(stream)), "mf_gated_residual_bwd")


def mf_adaln_bwd_workspace_size(T: int) -> int:
    return int(lib.mf_adaln_bwd_workspace_size(T))


def mf_adaln_modulate_bwd(dx_mod, x, mod, tok_sample, tok_mod, resid, T: int, S: int, hid: int,
                          eps: float, dx, dmod, workspace, ws_bytes: int, stream=None) -> None:
    _check(lib.mf_adaln_modulate_bwd(_ptr(dx_mod), _ptr(x), _ptr(mod), _ptr(tok_sample),
                                     _ptr(tok_mod), _ptr(resid), T, S, hid, eps, _ptr(dx),
                                     _ptr(dmod), _ptr(workspace), ws_bytes, _stream(stream)),
           "mf_adaln_modulate_bwd")


def mf_gated_residual(x, o, mod, tok_sample, tok_mod, T: int, S: int, hid: int, y,
                      stream=None) -> None:
    _check(lib.mf_gated_residual(_ptr(x), _ptr(o), _ptr(mod), _ptr(tok_sample), _ptr(tok_mod),
                                 T, S, hid, _ptr(y), _stream(stream)), "mf_gated_residual")


def mf_block_fwd(x, q, k, v, mod, cu_seqlens_d, cu_seqlens_h: np.ndarray, pos_ids, tok_sample,
                 tok_mod, S: int, H: int, D: int, rope_axes: int, base: float, eps: float, x_mod,
                 y, workspace, ws_bytes: int, stream=None) -> None:
    cu_h = np.ascontiguousarray(cu_seqlens_h, dtype=np.int32)
    _check(lib.mf_block_fwd(_ptr(x), _ptr(q), _ptr(k), _ptr(v), _ptr(mod), _ptr(cu_seqlens_d),
                            cu_h.ctypes.data_as(_P), _ptr(pos_ids), _ptr(tok_sample),
                            _ptr(tok_mod), S, H, D, rope_axes, base, eps, _ptr(x_mod), _ptr(y),
                            _ptr(workspace), ws_bytes, _stream(stream)), "mf_block_fwd")


def mf_workspace_size(T: int, H: int, D: int, with_rope: int) -> int:
    return int(lib.mf_workspace_size(T, H, D, with_rope))


def mf_get_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error word."""
    return int(lib.mf_get_error(_stream(stream)))


def mf_set_wait_limit_ns(ns: int) -> None:
    _check(lib.mf_set_wait_limit_ns(int(ns)), "mf_set_wait_limit_ns")


def mf_selftest_exp2_poly(x, y, n: int, stream=None) -> None:
    _check(lib.mf_selftest_exp2_poly(_ptr(x), _ptr(y), n, _stream(stream)), "mf_selftest_exp2_poly")


def mf_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(lib.mf_selftest_wait_timeout(int(limit_ns), _stream(stream)), "mf_selftest_wait_timeout")


def mf_set_attn_cta_pair(enable: int) -> None:
    _check(lib.mf_set_attn_cta_pair(int(enable)), "mf_set_attn_cta_pair")


def mf_set_linear_cta_pair(enable: int) -> None:
    _check(lib.mf_set_linear_cta_pair(int(enable)), "mf_set_linear_cta_pair")


def mf_set_conv_cta_pair(enable: int) -> None:
    _check(lib.mf_set_conv_cta_pair(int(enable)), "mf_set_conv_cta_pair")


def mf_set_attn_timing_events(start, stop) -> None:
    """``start`` / ``stop``: torch.cuda.Event objects (already recorded once, so
    that the CUDA event exists) or None to switch timing off."""
    def handle(ev):
        return None if ev is None else ev.cuda_event
    _check(lib.mf_set_attn_timing_events(handle(start), handle(stop)), "mf_set_attn_timing_events")


def mf_block_fwd_noalloc(x, q, k, v, mod, cu_seqlens_d, cu_seqlens_h: np.ndarray, pos_ids,
                         tok_sample, tok_mod, S: int, H: int, D: int, rope_axes: int, base: float,
                         eps: float, x_mod, y, stream=None) -> None:
    """mf_block_fwd for callers that cannot allocate device memory: the rotated
    Q and K live in the library's own fixed device array (see include/mf.h)."""
    cu_h = np.ascontiguousarray(cu_seqlens_h, dtype=np.int32)
    _check(lib.mf_block_fwd_noalloc(_ptr(x), _ptr(q), _ptr(k), _ptr(v), _ptr(mod),
                                    _ptr(cu_seqlens_d), cu_h.ctypes.data_as(_P), _ptr(pos_ids),
                                    _ptr(tok_sample), _ptr(tok_mod), S, H, D, rope_axes, base,
                                    eps, _ptr(x_mod), _ptr(y), _stream(stream)),
           "mf_block_fwd_noalloc")


class mf_cfg_pair(ctypes.Structure):
    _fields_ = [("cond", ctypes.c_int32), ("uncond", ctypes.c_int32)]


def mf_cfg_combine(v, descs, pairs, C: int, w: float, out, stream=None) -> None:
    """Packed classifier-free guidance: ``pairs`` are (cond, uncond) sample
    indices; ``out`` gets v_u + w (v_c - v_u) over each pair's image tokens."""
    arr = make_descs(descs)
    S = len(list(descs))
    pl = list(pairs)
    parr = (mf_cfg_pair * max(1, len(pl)))()
    for i, (c, u) in enumerate(pl):
        parr[i] = mf_cfg_pair(int(c), int(u))
    _check(lib.mf_cfg_combine(_ptr(v), ctypes.cast(arr, _P), S, ctypes.cast(parr, _P), len(pl),
                              C, w, _ptr(out), _stream(stream)), "mf_cfg_combine")


MF_ACT_NONE, MF_ACT_GELU = 0, 1


def mf_modality_linear(x, W, tok_mod, descs, K: int, N: int, out, act: int = MF_ACT_NONE,
                       stream=None) -> None:
    """out[t] = act(x[t] W[tok_mod[t]]^T): W is [2][N][K] (image weights first)."""
    arr = make_descs(descs)
    S = len(list(descs))
    _check(lib.mf_modality_linear(_ptr(x), _ptr(W), _ptr(tok_mod), ctypes.cast(arr, _P), S, K, N,
                                  act, _ptr(out), _stream(stream)), "mf_modality_linear")


def mf_mmdit_workspace_size(T: int, H: int, D: int, F: int) -> int:
    return int(lib.mf_mmdit_workspace_size(T, H, D, F))


def mf_mmdit_block_fwd(x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, descs, cu_seqlens_d,
                       cu_seqlens_h: np.ndarray, pos_ids, tok_sample, tok_mod, S: int, H: int,
                       D: int, F: int, rope_axes: int, base: float, eps: float, y, workspace,
                       ws_bytes: int, stream=None) -> None:
    arr = make_descs(descs)
    cu_h = np.ascontiguousarray(cu_seqlens_h, dtype=np.int32)
    _check(lib.mf_mmdit_block_fwd(_ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(Wo), _ptr(Wup),
                                  _ptr(Wdown), _ptr(mod_attn), _ptr(mod_mlp),
                                  ctypes.cast(arr, _P), _ptr(cu_seqlens_d), cu_h.ctypes.data_as(_P),
                                  _ptr(pos_ids), _ptr(tok_sample), _ptr(tok_mod), S, H, D, F,
                                  rope_axes, base, eps, _ptr(y), _ptr(workspace), ws_bytes,
                                  _stream(stream)), "mf_mmdit_block_fwd")


def mf_mmdit_bwd_workspace_size(T: int, S: int, H: int, D: int, F: int) -> int:
    return int(lib.mf_mmdit_bwd_workspace_size(T, S, H, D, F))


def mf_mmdit_block_bwd(dy, x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, descs, cu_seqlens_d,
                       cu_seqlens_h: np.ndarray, pos_ids, tok_sample, tok_mod, S: int, H: int,
                       D: int, F: int, rope_axes: int, base: float, eps: float, dx, dWq, dWk,
                       dWv, dWo, dWup, dWdown, dmod_attn, dmod_mlp, workspace, ws_bytes: int,
                       stream=None) -> None:
    arr = make_descs(descs)
    cu_h = np.ascontiguousarray(cu_seqlens_h, dtype=np.int32)
    _check(lib.mf_mmdit_block_bwd(_ptr(dy), _ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(Wo),
                                  _ptr(Wup), _ptr(Wdown), _ptr(mod_attn), _ptr(mod_mlp),
                                  ctypes.cast(arr, _P), _ptr(cu_seqlens_d), cu_h.ctypes.data_as(_P),
                                  _ptr(pos_ids), _ptr(tok_sample), _ptr(tok_mod), S, H, D, F,
                                  rope_axes, base, eps, _ptr(dx), _ptr(dWq), _ptr(dWk), _ptr(dWv),
                                  _ptr(dWo), _ptr(dWup), _ptr(dWdown), _ptr(dmod_attn),
                                  _ptr(dmod_mlp), _ptr(workspace), ws_bytes, _stream(stream)),
           "mf_mmdit_block_bwd")


def mf_gn_workspace_size(N: int, H: int, W: int, G: int) -> int:
    return int(lib.mf_gn_workspace_size(N, H, W, G))


def mf_group_norm_silu(x, gamma, beta, N: int, H: int, W: int, C: int, G: int, eps: float, y,
                       workspace, ws_bytes: int, stream=None) -> None:
    _check(lib.mf_group_norm_silu(_ptr(x), _ptr(gamma), _ptr(beta), N, H, W, C, G, eps, _ptr(y),
                                  _ptr(workspace), ws_bytes, _stream(stream)),
           "mf_group_norm_silu")


def mf_conv3x3(x, Wt, bias, residual, N: int, H: int, W: int, Cin: int, Cout: int, y,
               stream=None) -> None:
    _check(lib.mf_conv3x3(_ptr(x), _ptr(Wt), _ptr(bias), _ptr(residual), N, H, W, Cin, Cout,
                          _ptr(y), _stream(stream)), "mf_conv3x3")


def mf_vae_block_workspace_size(N: int, H: int, W: int, C: int, G: int) -> int:
    return int(lib.mf_vae_block_workspace_size(N, H, W, C, G))


def mf_vae_res_block(x, gamma1, beta1, W1, c1, gamma2, beta2, W2, c2, N: int, H: int, W: int,
                     C: int, G: int, eps: float, y, workspace, ws_bytes: int,
                     stream=None) -> None:
    _check(lib.mf_vae_res_block(_ptr(x), _ptr(gamma1), _ptr(beta1), _ptr(W1), _ptr(c1),
                                _ptr(gamma2), _ptr(beta2), _ptr(W2), _ptr(c2), N, H, W, C, G,
                                eps, _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)),
           "mf_vae_res_block")
