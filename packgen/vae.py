"""Synthetic inputs for the Mage-VAE conv block (fused normalization -
activation - residual chains).

The report gives the VAE's latent geometry (16x downsampling, 128 latent
channels) but not its stage widths; the shapes below are readings: decoder
stages of a 1024 x 1024 image at 1/8 resolution (128 x 128 pixels, 256
channels, 32 groups) and at 1/4 (256 x 256, 128 channels, 16 groups: eight
channels a group), plus a small ragged case for parity. Every array is drawn from ``numpy.random.default_rng(seed)``
in this order: x ~ N(0, 1) (bf16), W1 and W2 ~ N(0, 1) / sqrt(9 C) (bf16,
[C][3][3][C]), gamma1, beta1, gamma2, beta2 (fp32: 1 + 0.1 N(0,1) and
0.1 N(0,1)), c1 and c2 ~ 0.02 N(0, 1) (fp32). No arithmetic of the block lives
here.
"""

from __future__ import annotations

import dataclasses

import numpy as np

from .configs import bf16_bits_to_f32, f32_to_bf16_bits

VAE_CONFIGS = {
    "tiny": dict(N=2, H=9, W=13, C=64, G=8),
    "stage_1_8": dict(N=1, H=128, W=128, C=256, G=32),
    "stage_1_4": dict(N=1, H=256, W=256, C=128, G=16),
}


@dataclasses.dataclass
class VaeBlockInputs:
    name: str
    N: int
    H: int
    W: int
    C: int
    G: int
    eps: float
    seed: int
    x_bits: np.ndarray = None    # [N][H][W][C] bf16 bits
    W1_bits: np.ndarray = None   # [C][3][3][C] bf16 bits
    W2_bits: np.ndarray = None
    gamma1: np.ndarray = None    # [C] fp32
    beta1: np.ndarray = None
    gamma2: np.ndarray = None
    beta2: np.ndarray = None
    c1: np.ndarray = None        # [C] fp32 conv biases
    c2: np.ndarray = None

    def f32(self, name: str) -> np.ndarray:
        """A bf16 array as the float32 values it holds."""
        return bf16_bits_to_f32(getattr(self, name + "_bits"))


def make_vae_block(name: str = None, seed: int = None, **shape) -> VaeBlockInputs:
    """Inputs of one block: a named configuration, or N, H, W, C, G given."""
    spec = dict(VAE_CONFIGS[name]) if name is not None else {}
    spec.update(shape)
    N, H, W, C, G = (int(spec[k]) for k in ("N", "H", "W", "C", "G"))
    seed = 4000 + H + W + C if seed is None else seed
    rng = np.random.default_rng(seed)
    v = VaeBlockInputs(name=name or f"{N}x{H}x{W}x{C}", N=N, H=H, W=W, C=C, G=G, eps=1e-6,
                       seed=seed)

    def bf16(shape, scale=1.0):
        return f32_to_bf16_bits((rng.standard_normal(shape, dtype=np.float32)
                                 * np.float32(scale)).astype(np.float32))

    v.x_bits = bf16((N, H, W, C))
    v.W1_bits = bf16((C, 3, 3, C), 1.0 / np.sqrt(9.0 * C))
    v.W2_bits = bf16((C, 3, 3, C), 1.0 / np.sqrt(9.0 * C))
    f32 = lambda scale, shift=0.0: (shift + scale * rng.standard_normal(C)).astype(np.float32)  # noqa: E731
    v.gamma1, v.beta1 = f32(0.1, 1.0), f32(0.1)
    v.gamma2, v.beta2 = f32(0.1, 1.0), f32(0.1)
    v.c1, v.c2 = f32(0.02), f32(0.02)
    return v
