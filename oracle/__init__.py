"""CPU oracle for the packed joint-attention block -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package. The CUDA library never imports,
links or calls it, and it shares no code with the library: the only common
dependency is the seeded input generator ``packgen`` (random numbers and sample
descriptors, none of the block's arithmetic).

Sources (page title, then section). The pages give words, not formulas, for
every step of this path:
  [pack]  picx.dev "Mage-Flow" summary, Methodology > Native-Resolution MMDiT
          (NR-MMDiT), bullet "Native-resolution packing": images of different
          resolutions become variable-length latent token sequences, packed with
          variable-length text tokens under a fixed token budget; FlashAttention
          with per-sample cumulative offsets runs the attention.
  [rope]  gist.science "Resumo Tecnico: Mage-Flow", Metodologia > 2.
          Transformer de Difusao Multimodal de Resolucao Nativa, item
          "Empacotamento de Resolucao Nativa": per-sample 2D rotary embeddings
          with FlashAttention variable-length kernels.
  [edit]  picx.dev summary, Methodology > NR-MMDiT, bullet "Conditioning": for
          editing, source latents are concatenated with target latents under a
          3D RoPE whose frame dimension tells them apart.
  [norm]  picx.dev summary, Methodology > NR-MMDiT, first bullet: modality-
          specific normalization and joint self-attention.
  [fuse]  picx.dev summary, Methodology > Training Infrastructure: the fused
          chain in NR-MMDiT is adaptive normalization / RoPE / gating.
  [cfg]   picx.dev summary, Methodology > NR-MMDiT, bullet "Packed CFG
          inference": conditional and unconditional branches in one forward.
  [vae], [vfuse] (``vae_oracle``) picx.dev summary, Methodology > Mage-VAE and
          > Training Infrastructure: the fully convolutional VAE's repeated
          blocks and their fused normalization - activation - residual chains.

Where the pages are silent the oracle takes one stated reading (RoPE split and
base, text positions, LayerNorm eps, modulation form); each reading is named at
the function that uses it.

Pins: ``tests/test_oracle_pins.py`` checks every function against closed forms,
invariants, a library routine (torch SDPA in fp64), a pure-Python brute force
(``oracle.brute``) and hand-derived fixtures in ``tests/golden/``. The reading
choices themselves (pair layout, axis split, eps, text positions) have no worked
example on the pages: against the pages they are "parity unpinned"; they are
pinned only against the stated reading.
"""

from .mf_oracle import (  # noqa: F401
    MOD_IMG,
    MOD_TXT,
    adaln_modulate,
    adaln_modulate_bwd,
    adaln_params,
    adaln_params_bwd,
    block_bwd,
    block_fwd,
    cfg_combine,
    gated_residual,
    gated_residual_bwd,
    gelu_tanh,
    gelu_tanh_bwd,
    layer_norm_rows,
    mmdit_block_bwd,
    mmdit_block_fwd,
    modality_linear,
    modality_linear_bwd,
    pack_build,
    rope_apply,
    rope_bwd,
    rope_pair_angles,
    rope_split,
    store_bf16,
    useful_attention_flops,
    varlen_attention,
    varlen_attention_bwd,
)
from .vae_oracle import (  # noqa: F401
    conv3x3,
    group_norm,
    group_norm_silu,
    silu,
    vae_block_flops,
    vae_res_block,
)
