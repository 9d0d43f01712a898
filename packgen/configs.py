"""Synthetic workloads shaped like the Mage-Flow report's packs.

The report's datasets and checkpoints are not used: every array here is drawn
from ``numpy.random.default_rng(seed)``. Grid sizes follow the report's latent
geometry (Mage-Flow summary on picx.dev, Methodology > Mage-VAE: latents are
16x downsampled, 128 channels), so a 1024x1024 image is a 64x64 token grid, a
2048x2048 image 128x128 and a 512x2048 image 32x128.

Recipe (the same for every workload):
  * seed = 1000 + workload index;
  * draw order: text lengths (integers, uniform, inclusive bounds), then x, q,
    k, v (standard normal float32, rounded to bf16 round-to-nearest-even),
    then the conditioning vectors c ~ N(0,1) [S][128] and the linear map
    W ~ 0.02 * N(0,1) [128][6*hid] (both float32).

Only shapes and random numbers live here; the arithmetic of the block is in the
oracle and in the CUDA library, which share none of it.
"""

from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np

COND_DIM = 128  # size of the per-sample conditioning vector in every workload


@dataclasses.dataclass(frozen=True)
class SampleDesc:
    """One sample of a pack: ``frames`` latent grids of ``grid_h x grid_w``
    tokens followed by ``n_text`` text tokens. ``is_dummy`` marks the padding
    segment that fills a training pack up to its token budget."""

    frames: int
    grid_h: int
    grid_w: int
    n_text: int
    is_dummy: int = 0

    def as_tuple(self):
        return (self.frames, self.grid_h, self.grid_w, self.n_text, self.is_dummy)


def token_count(descs: Sequence[SampleDesc]) -> int:
    """Total number of tokens the descriptors occupy (used to size arrays)."""
    return int(sum(d.frames * d.grid_h * d.grid_w + d.n_text for d in descs))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); returns the
    16-bit patterns. Inputs here are finite, so NaN handling is not needed."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact float32 values of bfloat16 bit patterns."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Workload:
    index: int
    name: str
    descs: List[SampleDesc]
    H: int
    D: int
    rope_axes: int
    budget: int
    seed: int
    base: float = 10000.0
    eps: float = 1e-6
    # bf16 bit patterns (uint16) and their exact float32 values
    x_bits: Optional[np.ndarray] = None  # [T][hid]
    q_bits: Optional[np.ndarray] = None  # [T][H][D]
    k_bits: Optional[np.ndarray] = None
    v_bits: Optional[np.ndarray] = None
    c: Optional[np.ndarray] = None  # [S][COND_DIM] float32
    W: Optional[np.ndarray] = None  # [COND_DIM][6*hid] float32
    # packed-CFG packs: (conditional, unconditional) sample index pairs
    cfg_pairs: List[tuple] = dataclasses.field(default_factory=list)

    @property
    def hid(self) -> int:
        return self.H * self.D

    @property
    def S(self) -> int:
        return len(self.descs)

    @property
    def T(self) -> int:
        return token_count(self.descs)

    def f32(self, name: str) -> np.ndarray:
        return bf16_bits_to_f32(getattr(self, name + "_bits"))


# Workload table. ``text`` entries are either fixed lengths or (lo, hi) ranges
# drawn uniformly (inclusive) in the order listed.
CONFIGS = {
    1: dict(name="tiny pack, 544 tokens, 2 heads x 64",
            H=2, D=64, rope_axes=2, budget=0,
            samples=[(1, 16, 16, 20), (1, 8, 32, 12)]),
    2: dict(name="native-resolution training pack, 16384-token budget, 24 heads x 128",
            H=24, D=128, rope_axes=2, budget=16384,
            samples=[(1, 64, 64, (64, 256)), (1, 32, 128, (64, 256)),
                     (1, 48, 48, (64, 256)), (1, 32, 32, (64, 256))],
            pad_to_budget=True),
    3: dict(name="packed CFG at 1024x1024, 8464 tokens, 24 heads x 128",
            H=24, D=128, rope_axes=2, budget=0,
            samples=[(1, 64, 64, 256), (1, 64, 64, 16)],
            cfg_pairs=[(0, 1)]),  # (conditional, unconditional) branch samples
    4: dict(name="edit pack, source+target 64x64, 3D RoPE, 16896 tokens, 24 heads x 128",
            H=24, D=128, rope_axes=3, budget=0,
            samples=[(2, 64, 64, 256), (2, 64, 64, 256)]),
    5: dict(name="large pack, 32768-token budget, 24 heads x 128",
            H=24, D=128, rope_axes=2, budget=32768,
            samples=[(1, 128, 128, 512), (1, 128, 32, (128, 512)),
                     (1, 128, 32, (128, 512)), (1, 32, 128, (128, 512))]),
}


def _draw_normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def draw_grad_bits(seed: int, shape) -> np.ndarray:
    """Seeded standard-normal bf16 bits, the upstream gradient (dO) of the
    backward tests and bench."""
    return _draw_normal_bf16(np.random.default_rng(seed), shape)


def fill_arrays(w: Workload, rng: np.random.Generator) -> Workload:
    T, H, D, hid, S = w.T, w.H, w.D, w.hid, w.S
    w.x_bits = _draw_normal_bf16(rng, (T, hid))
    w.q_bits = _draw_normal_bf16(rng, (T, H, D))
    w.k_bits = _draw_normal_bf16(rng, (T, H, D))
    w.v_bits = _draw_normal_bf16(rng, (T, H, D))
    w.c = rng.standard_normal((S, COND_DIM), dtype=np.float32)
    w.W = (rng.standard_normal((COND_DIM, 6 * hid), dtype=np.float32)
           * np.float32(0.02)).astype(np.float32)
    return w


def make_workload(index: int, with_arrays: bool = True, seed: Optional[int] = None) -> Workload:
    """Build workload ``index`` (1..5) with its seeded arrays."""
    spec = CONFIGS[index]
    seed = 1000 + index if seed is None else seed
    rng = np.random.default_rng(seed)
    descs = []
    for (f, gh, gw, text) in spec["samples"]:
        if isinstance(text, tuple):
            n_text = int(rng.integers(text[0], text[1] + 1))
        else:
            n_text = int(text)
        descs.append(SampleDesc(f, gh, gw, n_text))
    if spec.get("pad_to_budget"):
        fill = spec["budget"] - token_count(descs)
        if fill > 0:
            descs.append(SampleDesc(0, 0, 0, fill, 1))
    w = Workload(index=index, name=spec["name"], descs=descs, H=spec["H"], D=spec["D"],
                 rope_axes=spec["rope_axes"], budget=spec["budget"], seed=seed,
                 cfg_pairs=list(spec.get("cfg_pairs", [])))
    if with_arrays:
        fill_arrays(w, rng)
    return w


def make_random_pack(seed: int, S: int, H: int, D: int, rope_axes: int,
                     max_grid: int = 6, max_text: int = 8,
                     descs: Optional[Sequence[SampleDesc]] = None) -> Workload:
    """A small random pack for edge cases and brute-force checks. ``descs``
    overrides the drawn sample list."""
    rng = np.random.default_rng(seed)
    if descs is None:
        descs = []
        for _ in range(S):
            frames = int(rng.integers(1, 3)) if rope_axes == 3 else 1
            gh = int(rng.integers(0, max_grid + 1))
            gw = int(rng.integers(0, max_grid + 1))
            descs.append(SampleDesc(frames, gh, gw, int(rng.integers(0, max_text + 1))))
    w = Workload(index=0, name=f"random pack seed {seed}", descs=list(descs), H=H, D=D,
                 rope_axes=rope_axes, budget=0, seed=seed)
    return fill_arrays(w, rng)
