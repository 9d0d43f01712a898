"""Pins of the Mage-VAE block's oracle (``oracle/vae_oracle.py``), checked
without a GPU against library routines (torch's fp64 group_norm, silu and
conv2d: NCHW, with the same padding and cross-correlation convention), a
pure-Python brute force, closed-form cases (identity and shifting kernels, a
zero second conv) and invariants (GroupNorm moments); then planted mistakes in
copies of the oracle, each of which some pin must catch."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import vae_oracle as vo
from packgen import make_vae_block


def _nchw(a):
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.float64).transpose(0, 3, 1, 2)))


def _nhwc(t):
    return t.numpy().transpose(0, 2, 3, 1)


def _rand(seed, shape, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ------------------------------------------------------------------ pins
def pin_group_norm_library(gn=vo.group_norm):
    x = _rand(1, (2, 5, 7, 24))
    g, b = 1 + 0.1 * _rand(2, 24), 0.1 * _rand(3, 24)
    ref = F.group_norm(_nchw(x), 6, torch.from_numpy(g), torch.from_numpy(b), eps=1e-6)
    return np.abs(gn(x, g, b, 6, 1e-6) - _nhwc(ref)).max() < 1e-12


def pin_group_norm_moments(gn=vo.group_norm):
    x = 3.0 + 2.0 * _rand(4, (2, 6, 4, 32))
    y = gn(x, np.ones(32), np.zeros(32), 4, 0.0).reshape(2, 24, 4, 8)
    return (np.abs(y.mean(axis=(1, 3))).max() < 1e-12 and
            np.abs(y.var(axis=(1, 3)) - 1).max() < 1e-12)


def pin_silu_library(s=vo.silu):
    x = _rand(5, 1000, 4.0)
    return np.abs(s(x) - F.silu(torch.from_numpy(x)).numpy()).max() < 1e-14


def pin_conv_library(conv=vo.conv3x3):
    x = _rand(6, (2, 6, 9, 16))
    W = _rand(7, (24, 3, 3, 16), 0.1)
    bias, res = _rand(8, 24), _rand(9, (2, 6, 9, 24))
    ref = F.conv2d(_nchw(x), torch.from_numpy(W.transpose(0, 3, 1, 2).copy()),
                   torch.from_numpy(bias), padding=1)
    return np.abs(conv(x, W, bias, res) - (_nhwc(ref) + res)).max() < 1e-11


def pin_conv_brute_force(conv=vo.conv3x3):
    x = _rand(10, (1, 3, 4, 2))
    W = _rand(11, (3, 3, 3, 2))
    got = conv(x, W)
    for h in range(3):
        for w in range(4):
            for o in range(3):
                acc = 0.0
                for dy in range(3):
                    for dx in range(3):
                        hh, ww = h + dy - 1, w + dx - 1
                        if 0 <= hh < 3 and 0 <= ww < 4:
                            for i in range(2):
                                acc += x[0, hh, ww, i] * W[o, dy, dx, i]
                if abs(got[0, h, w, o] - acc) > 1e-12:
                    return False
    return True


def pin_conv_identity_and_shift(conv=vo.conv3x3):
    x = _rand(12, (1, 4, 5, 3))
    eye = np.zeros((3, 3, 3, 3))
    eye[:, 1, 1, :] = np.eye(3)
    shift = np.zeros((3, 3, 3, 3))
    shift[:, 1, 2, :] = np.eye(3)  # tap (dy, dx) = (1, 2) reads pixel (h, w + 1)
    expect = np.zeros_like(x)
    expect[:, :, :-1] = x[:, :, 1:]  # zero padding beyond the right edge
    return (np.abs(conv(x, eye) - x).max() == 0 and
            np.abs(conv(x, shift) - expect).max() == 0)


def pin_block_zero_second_conv(block=vo.vae_res_block):
    v = make_vae_block(N=1, H=5, W=6, C=16, G=4, seed=13)
    y = block(v.f32("x"), v.gamma1, v.beta1, v.f32("W1"), v.c1, v.gamma2, v.beta2,
              np.zeros((16, 3, 3, 16)), np.zeros(16), 4, v.eps)
    return np.array_equal(y, v.f32("x").astype(np.float64))


def pin_block_composition(block=vo.vae_res_block):
    """Unrounded, the block is the composition of the library routines."""
    v = make_vae_block(N=2, H=4, W=7, C=16, G=4, seed=14)
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))  # noqa: E731
    w = lambda name: t(v.f32(name).transpose(0, 3, 1, 2).copy())  # noqa: E731
    x = _nchw(v.f32("x"))
    a1 = F.silu(F.group_norm(x, 4, t(v.gamma1), t(v.beta1), eps=v.eps))
    h = F.conv2d(a1, w("W1"), t(v.c1), padding=1)
    a2 = F.silu(F.group_norm(h, 4, t(v.gamma2), t(v.beta2), eps=v.eps))
    ref = _nhwc(x + F.conv2d(a2, w("W2"), t(v.c2), padding=1))
    got = block(v.f32("x"), v.gamma1, v.beta1, v.f32("W1"), v.c1, v.gamma2, v.beta2,
                v.f32("W2"), v.c2, 4, v.eps, store=lambda a: np.asarray(a, np.float64))
    return np.abs(got - ref).max() < 1e-11


PINS = [pin_group_norm_library, pin_group_norm_moments, pin_silu_library, pin_conv_library,
        pin_conv_brute_force, pin_conv_identity_and_shift, pin_block_zero_second_conv,
        pin_block_composition]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_vae_oracle_pin(pin):
    assert pin()


def test_oracle_exports_the_vae_functions():
    assert oracle.vae_res_block is vo.vae_res_block and oracle.conv3x3 is vo.conv3x3
    assert oracle.vae_block_flops(1, 128, 128, 256) == 4.0 * 9 * 256 * 256 * 128 * 128


# ------------------------------------------------------------------ mutants
def _gn_channel_groups_strided(x, gamma, beta, G, eps=1e-6):
    # groups of every G-th channel instead of consecutive channels
    x = np.asarray(x, np.float64)
    N, H, W, C = x.shape
    perm = np.arange(C).reshape(C // G, G).T.reshape(-1)
    inv = np.argsort(perm)
    return vo.group_norm(x[..., perm], np.asarray(gamma)[perm], np.asarray(beta)[perm], G,
                         eps)[..., inv]


def _gn_sample_var(x, gamma, beta, G, eps=1e-6):
    x = np.asarray(x, np.float64)
    N, H, W, C = x.shape
    xg = x.reshape(N, H * W, G, C // G)
    mean = xg.mean(axis=(1, 3), keepdims=True)
    var = xg.reshape(N, -1, G, C // G).transpose(0, 2, 1, 3).reshape(N, G, -1).var(
        axis=2, ddof=1)[:, None, :, None]
    return ((xg - mean) / np.sqrt(var + eps)).reshape(N, H, W, C) * gamma + beta


def _silu_sigmoid_only(x):
    x = np.asarray(x, np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def _conv_flipped_taps(x, Wt, bias=None, residual=None):
    return vo.conv3x3(x, np.asarray(Wt)[:, ::-1, ::-1, :], bias, residual)


def _conv_weight_untransposed(x, Wt, bias=None, residual=None):
    Wt = np.asarray(Wt)
    return vo.conv3x3(x, Wt.transpose(3, 1, 2, 0), bias, residual)


def _conv_dropped_bias(x, Wt, bias=None, residual=None):
    return vo.conv3x3(x, Wt, None, residual)


def _block_no_skip(x, g1, b1, W1, c1, g2, b2, W2, c2, G, eps=1e-6, store=oracle.store_bf16):
    return vo.vae_res_block(x, g1, b1, W1, c1, g2, b2, W2, c2, G, eps, store) - np.asarray(
        x, np.float64)


MUTANTS = [
    ("group norm over strided channel groups", "group_norm", _gn_channel_groups_strided,
     [pin_group_norm_library]),
    ("group norm with the sample variance", "group_norm", _gn_sample_var,
     [pin_group_norm_library, pin_group_norm_moments]),
    ("SiLU without the x factor", "silu", _silu_sigmoid_only, [pin_silu_library]),
    ("conv with flipped taps", "conv3x3", _conv_flipped_taps,
     [pin_conv_library, pin_conv_brute_force, pin_conv_identity_and_shift]),
    ("conv weights read [Cin][..][Cout]", "conv3x3", _conv_weight_untransposed,
     [pin_conv_library, pin_conv_brute_force]),
    ("conv without its bias", "conv3x3", _conv_dropped_bias, [pin_conv_library]),
    ("block without the identity skip", "vae_res_block", _block_no_skip,
     [pin_block_zero_second_conv, pin_block_composition]),
]


@pytest.mark.parametrize("name,target,mutant,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_vae_mutant_is_caught(name, target, mutant, pins):
    """Each listed pin runs against the mutant in place of the oracle function;
    at least one fails (or cannot run on it)."""
    caught = False
    for pin in pins:
        try:
            ok = pin(mutant)
        except ValueError:  # the mutant cannot even take the pin's shapes
            ok = False
        caught = caught or not ok
    assert caught, f"no pin caught: {name}"
