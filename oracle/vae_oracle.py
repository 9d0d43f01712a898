"""Plain fp64 NumPy definition of the Mage-VAE conv block's fused chains.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): slow, obviously correct,
no blocking or fusion beyond what each definition states.

Source (page title, then section):
  [vae]   picx.dev "Mage-Flow" summary, Methodology > Mage-VAE, "Architecture":
          the decoder is a fully convolutional one-step pixel diffusion model
          (no global attention) built from stacked convolutional diffusion
          blocks; the encoder is its dual; latents are 16x downsampled with 128
          channels.
  [vfuse] picx.dev summary, Methodology > Training Infrastructure: the stack's
          CUDA kernel fusion fuses the normalization - activation - residual
          chains of Mage-VAE's repeated blocks.
The pages give neither the block's wiring nor its widths. Reading taken (the
residual block of diffusion conv nets): GroupNorm with affine parameters, SiLU,
3x3 convolution (stride 1, zero padding 1, with bias), twice, plus the identity
skip:
    h = conv3x3(SiLU(GN(x; gamma1, beta1)); W1, c1)
    y = x + conv3x3(SiLU(GN(h; gamma2, beta2)); W2, c2)
Layout NHWC ([N][H][W][C], channels innermost); GroupNorm over each sample's
(H, W, C / G channels of the group) with the population variance; conv weights
[Cout][3][3][Cin] (tap (dy, dx) reads input pixel (h + dy - 1, w + dx - 1)).
Inputs arrive as float32 arrays holding exact bf16 (activations, weights) or
fp32 (GroupNorm affine parameters, biases) values; every computation is float64.
"""

from __future__ import annotations

import numpy as np

from .mf_oracle import store_bf16


def silu(x) -> np.ndarray:
    """SiLU (swish): x * sigmoid(x) = x / (1 + exp(-x))."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def group_norm(x, gamma, beta, G: int, eps: float = 1e-6) -> np.ndarray:
    """GroupNorm of an NHWC tensor: the C channels are G consecutive groups of
    C / G; each (sample, group) is normalised over its H x W x C / G elements
    (population variance), then channel c is scaled by gamma[c] and shifted by
    beta[c]."""
    x = np.asarray(x, dtype=np.float64)
    N, H, W, C = x.shape
    if C % G:
        raise ValueError("C must be a multiple of G")
    xg = x.reshape(N, H * W, G, C // G)
    mean = xg.mean(axis=(1, 3), keepdims=True)
    var = ((xg - mean) ** 2).mean(axis=(1, 3), keepdims=True)
    xn = ((xg - mean) / np.sqrt(var + eps)).reshape(N, H, W, C)
    return xn * np.asarray(gamma, dtype=np.float64) + np.asarray(beta, dtype=np.float64)


def group_norm_silu(x, gamma, beta, G: int, eps: float = 1e-6) -> np.ndarray:
    """The fused normalization - activation step: SiLU(GroupNorm(x))."""
    return silu(group_norm(x, gamma, beta, G, eps))


def conv3x3(x, Wt, bias=None, residual=None) -> np.ndarray:
    """3x3 convolution, stride 1, zero padding 1, on NHWC: out[n, h, w, o] =
    sum over dy, dx in {0, 1, 2} and input channels i of
    x[n, h + dy - 1, w + dx - 1, i] * Wt[o, dy, dx, i] (zero outside the image),
    plus bias[o] and the residual[n, h, w, o] when given. Each of the nine taps
    is one matrix product over the channels."""
    x = np.asarray(x, dtype=np.float64)
    Wt = np.asarray(Wt, dtype=np.float64)
    N, H, W, _ = x.shape
    Cout = Wt.shape[0]
    xp = np.pad(x, ((0, 0), (1, 1), (1, 1), (0, 0)))
    out = np.zeros((N, H, W, Cout))
    for dy in range(3):
        for dx in range(3):
            out += xp[:, dy:dy + H, dx:dx + W, :] @ Wt[:, dy, dx, :].T
    if bias is not None:
        out += np.asarray(bias, dtype=np.float64)
    if residual is not None:
        out += np.asarray(residual, dtype=np.float64)
    return out


def vae_res_block(x, gamma1, beta1, W1, c1, gamma2, beta2, W2, c2, G: int,
                  eps: float = 1e-6, store=store_bf16) -> np.ndarray:
    """One conv block of the reading above. Every intermediate (the two
    SiLU(GN(.)) activations and h) is stored in bf16 (``store``), as the GPU
    chain stores them; the output y is returned unrounded (float64)."""
    a1 = store(group_norm_silu(x, gamma1, beta1, G, eps))
    h = store(conv3x3(a1, W1, c1))
    a2 = store(group_norm_silu(h, gamma2, beta2, G, eps))
    return conv3x3(a2, W2, c2, residual=x)


def vae_block_flops(N: int, H: int, W: int, C: int) -> float:
    """FLOPs of the block's two convolutions: 2 x (2 x 9 x C x C per pixel)."""
    return 2.0 * 2.0 * 9.0 * C * C * N * H * W
