"""Seeded synthetic workloads for Sliding Tile Attention (STA) forward.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark.  It holds only workload shapes and seeded random inputs: none of the
method's arithmetic lives here.

Shapes follow the pages on "Fast Video Generation with Sliding Tile Attention":
the HunyuanVideo 720P / 5 s latent is (30, 48, 80) tokens (page 1, experiment
design; page 3, reply on input resolution) and the authors' tile is (6, 8, 8)
(page 3, reply on input resolution).  The other shapes are small, 2D and
long-video variants of the same workload.

Input recipe (the same on every machine):
  * for each (batch b, head h) a CPU ``torch.Generator`` is seeded with
    ``head_seed(seed, b, h)``; it draws fp32 ``randn(L, d)`` for q, then k,
    then v, in raster token order, and each is rounded to bf16 (round to
    nearest even);
  * per-head windows of the "perhead" workload come from splitmix64 seeded with
    5: head i takes ``WINDOW_CHOICES[(next() >> 33) % 4]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Sequence, Tuple

import torch

Dim3 = Tuple[int, int, int]

MASK64 = (1 << 64) - 1

# Window choices of the per-head workload, in tiles.  (5, 6, 10) is listed by the
# workload description as "dense"; on the 8x6x10 tile grid it is dense in H and W
# only (5 of 8 temporal tiles).  It is used literally.
WINDOW_CHOICES: Tuple[Dim3, ...] = ((1, 3, 3), (3, 3, 3), (3, 5, 5), (5, 6, 10))


def splitmix64_stream(seed: int):
    """Yield successive splitmix64 outputs (Steele, Lea, Flood 2014)."""
    state = seed & MASK64
    while True:
        state = (state + 0x9E3779B97F4A7C15) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        yield z ^ (z >> 31)


def perhead_windows(heads: int, seed: int = 5) -> List[Dim3]:
    gen = splitmix64_stream(seed)
    return [WINDOW_CHOICES[(next(gen) >> 33) % 4] for _ in range(heads)]


@dataclass(frozen=True)
class StaConfig:
    name: str
    batch: int
    heads: int
    d: int
    grid: Dim3        # latent (T, H, W) in tokens
    tile: Dim3        # (tt, th, tw) in tokens
    windows: Tuple[Dim3, ...] = field(default_factory=tuple)  # per head, in tiles

    @property
    def L(self) -> int:
        return self.grid[0] * self.grid[1] * self.grid[2]

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def ntile(self) -> int:
        return self.tile[0] * self.tile[1] * self.tile[2]


def _cfg(name, batch, heads, d, grid, tile, windows) -> StaConfig:
    if len(windows) == 1:
        windows = list(windows) * heads
    return StaConfig(name, batch, heads, d, tuple(grid), tuple(tile), tuple(tuple(w) for w in windows))


CONFIGS = {
    # 256 tokens, 2x2x2 tile grid; head 0 block-diagonal, head 1 window larger than the grid.
    "tiny": _cfg("tiny", 1, 2, 64, (4, 8, 8), (2, 4, 4), [(1, 1, 1), (3, 3, 3)]),
    # 11520 tokens, 2x3x5 tile grid.
    "small": _cfg("small", 1, 4, 128, (12, 24, 40), (6, 8, 8), [(1, 3, 3)]),
    # HunyuanVideo 720P 5 s latent: 115200 tokens, 5x6x10 tile grid.
    "hunyuan": _cfg("hunyuan", 1, 24, 128, (30, 48, 80), (6, 8, 8), [(3, 3, 3)]),
    # image-shaped (T = 1): 16384 tokens, 1x16x8 tile grid.
    "image2d": _cfg("image2d", 2, 24, 128, (1, 128, 128), (1, 8, 16), [(1, 5, 3)]),
    # long video with per-head windows: 184320 tokens, 8x6x10 tile grid.
    "perhead": _cfg("perhead", 1, 24, 128, (48, 48, 80), (6, 8, 8), perhead_windows(24, 5)),
}


def custom_config(name: str, batch: int, heads: int, d: int, grid: Sequence[int],
                  tile: Sequence[int], windows: Sequence[Sequence[int]]) -> StaConfig:
    return _cfg(name, batch, heads, d, grid, tile, windows)


def head_seed(seed: int, b: int, h: int) -> int:
    """Seed of the CPU generator for one (batch, head) slice."""
    return (seed * 1_000_003 + b * 10_007 + h * 101 + 17) & 0x7FFFFFFFFFFFFFFF


def make_head(cfg: StaConfig, seed: int, b: int, h: int):
    """q, k, v of one (batch, head) slice: bf16 tensors [L, d] in raster order (CPU)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(head_seed(seed, b, h))
    out = []
    for _ in range(3):
        x = torch.randn(cfg.L, cfg.d, generator=g, dtype=torch.float32)
        out.append(x.to(torch.bfloat16))
    return tuple(out)


def make_qkv(cfg: StaConfig, seed: int = 0):
    """q, k, v as bf16 CPU tensors [B, heads, L, d] in raster order."""
    shape = (cfg.batch, cfg.heads, cfg.L, cfg.d)
    q = torch.empty(shape, dtype=torch.bfloat16)
    k = torch.empty(shape, dtype=torch.bfloat16)
    v = torch.empty(shape, dtype=torch.bfloat16)
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            qh, kh, vh = make_head(cfg, seed, b, h)
            q[b, h].copy_(qh)
            k[b, h].copy_(kh)
            v[b, h].copy_(vh)
    return q, k, v


def sample_rows(cfg: StaConfig, seed: int, n_random: int = 128) -> List[int]:
    """Raster-order query rows for sampled parity on large workloads.

    All rows of the tile at tile coordinate (0, 0, 0), of an interior tile and
    of the last tile, plus ``n_random`` seeded random rows.
    """
    T, H, W = cfg.grid
    tt, th, tw = cfg.tile
    nT, nH, nW = T // tt, H // th, W // tw

    def tile_rows(a):
        rows = []
        for t in range(a[0] * tt, a[0] * tt + tt):
            for hh in range(a[1] * th, a[1] * th + th):
                for w in range(a[2] * tw, a[2] * tw + tw):
                    rows.append((t * H + hh) * W + w)
        return rows

    rows = set(tile_rows((0, 0, 0)))
    rows |= set(tile_rows((nT // 2, nH // 2, nW // 2)))
    rows |= set(tile_rows((nT - 1, nH - 1, nW - 1)))
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + 4242)
    rows |= set(torch.randint(0, cfg.L, (n_random,), generator=g).tolist())
    return sorted(rows)
