"""Seeded synthetic inputs for the packed joint-attention block.

This package only draws random numbers and lays out sample descriptors. It holds
none of the block's arithmetic (no normalisation, rotation, attention or gating),
so the CPU oracle under ``oracle/`` and the CUDA path under
``resolution_packed_diffusion_b200/`` can both consume it without sharing code.
"""

from .configs import (  # noqa: F401
    CONFIGS,
    COND_DIM,
    SampleDesc,
    Workload,
    bf16_bits_to_f32,
    draw_grad_bits,
    f32_to_bf16_bits,
    make_workload,
    make_random_pack,
    token_count,
)
from .vae import VAE_CONFIGS, VaeBlockInputs, make_vae_block  # noqa: F401,E402
