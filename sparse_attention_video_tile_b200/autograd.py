"""Sliding Tile Attention with autograd, for finetuning.

The forward keeps each row's log-sum-exp; the backward gives dq, dk and dv over
the same tile windows ("Fast Video Generation with Sliding Tile Attention",
abstract and "Method details": attention restricted to a sliding window of whole
tiles; the review replies describe finetuning with it).  Every step runs in the
library's CUDA kernels through the C ABI:

    forward   raster q, k, v --tile reorder--> tiled --sta_attention_fwd_lse--> tiled out, lse
              tiled out --tile unorder--> raster out
    backward  raster dout --tile reorder--> tiled --sta_attention_bwd--> tiled dq, dk, dv
              --tile unorder--> raster dq, dk, dv

Raster tensors are either [B, heads, L, d] (``token_major=False``) or the
token-major [B, L, heads, d] (``token_major=True``), where the transposes are
part of the reorders.  The tiled q, k, v, output and log-sum-exp are kept for
the backward.  Tiles must hold a multiple of 128 tokens and the grid must be a
tile multiple (the backward kernel's blocking).  The backward is not itself
differentiable: a second derivative raises.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch
from torch.autograd.function import once_differentiable

from . import (sta_attention_bwd, sta_attention_fwd_lse, sta_tile_reorder, sta_tile_reorder_tokens,
               sta_tile_unorder, sta_tile_unorder_tokens)


def _to_tiled(x, grid, tile, token_major: bool):
    if token_major:
        b, n, h, d = x.shape
        t = torch.empty((b, h, n, d), dtype=x.dtype, device=x.device)
        sta_tile_reorder_tokens(x, t, grid, tile)
    else:
        t = torch.empty_like(x)
        sta_tile_reorder(x, t, grid, tile)
    return t


def _from_tiled(t, grid, tile, token_major: bool):
    if token_major:
        b, h, n, d = t.shape
        x = torch.empty((b, n, h, d), dtype=t.dtype, device=t.device)
        sta_tile_unorder_tokens(t, x, grid, tile)
    else:
        x = torch.empty_like(t)
        sta_tile_unorder(t, x, grid, tile)
    return x


class STAttentionFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, grid, tile, windows, scale, token_major):
        qt, kt, vt = (_to_tiled(x.contiguous(), grid, tile, token_major) for x in (q, k, v))
        ot = torch.empty_like(qt)
        b, h, n, _ = qt.shape
        lse = torch.empty((b, h, n), dtype=torch.float32, device=qt.device)
        sta_attention_fwd_lse(qt, kt, vt, ot, lse, grid, tile, windows, scale)
        ctx.save_for_backward(qt, kt, vt, ot, lse)
        ctx.sta_args = (grid, tile, windows, scale, token_major)
        return _from_tiled(ot, grid, tile, token_major)

    @staticmethod
    @once_differentiable
    def backward(ctx, dout):
        qt, kt, vt, ot, lse = ctx.saved_tensors
        grid, tile, windows, scale, token_major = ctx.sta_args
        dot = _to_tiled(dout.to(torch.bfloat16).contiguous(), grid, tile, token_major)
        dq, dk, dv = (torch.empty_like(qt) for _ in range(3))
        sta_attention_bwd(qt, kt, vt, ot, dot, lse, dq, dk, dv, grid, tile, windows, scale)
        grads = tuple(_from_tiled(g, grid, tile, token_major) for g in (dq, dk, dv))
        return grads + (None, None, None, None, None)


def sta_attention(q, k, v, grid, tile, window_per_head: Sequence, scale: Optional[float] = None,
                  token_major: bool = False):
    """STA forward with a backward: bf16 CUDA tensors in raster order, [B, heads, L, d]
    or, with ``token_major``, [B, L, heads, d]; output in the same layout."""
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    return STAttentionFunction.apply(q, k, v, tuple(grid), tuple(tile),
                                     [tuple(w) for w in window_per_head], float(scale), bool(token_major))
