"""Sharded STA forward over several GPUs (one process per GPU).

(batch, head) pairs of Sliding Tile Attention are independent and each head has
its own window, so heads split across ranks with no exchange inside attention:
every rank runs the CUDA path on its contiguous range of heads.

Two entry points:

* ``sta_forward_head_sharded``: every rank holds the whole q, k, v; it computes
  its heads, and an all-gather gives every rank the full output.
* ``sta_forward_sequence_sharded``: every rank holds a contiguous range of the
  tokens (raster order) for all heads, in the token-major [B, L, heads, d]
  layout of a sequence-parallel video transformer.  One all-to-all turns token
  shards into head shards (all tokens, the rank's heads), the rank runs the
  CUDA path on them, and a second all-to-all returns the rank's tokens for all
  heads (the Ulysses scheme of sequence parallelism).

This module holds host logic only: the partitions, the collectives (NCCL over
NVLink on B200; any torch.distributed backend works for the host logic) with
the packing around them, and the calls into the CUDA path.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple


def _balanced_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if n < 0:
        raise ValueError("the count must be non-negative")
    base, extra = divmod(n, world)
    a = rank * base + min(rank, extra)
    return a, a + base + (1 if rank < extra else 0)


def head_range(heads: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous range [h0, h1) of the heads owned by `rank`: the first
    heads % world ranks take one head more than the others."""
    return _balanced_range(heads, world, rank)


def token_range(L: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous range [t0, t1) of the raster-order tokens held by `rank` in the
    sequence-sharded layout, split like the heads."""
    return _balanced_range(L, world, rank)


def head_counts(heads: int, world: int) -> List[int]:
    return [b - a for a, b in (head_range(heads, world, r) for r in range(world))]


def gather_heads(local, heads: int, group=None):
    """All-gathers per-rank head slices [B, h1 - h0, L, d] (contiguous ranges in rank
    order, as `head_range` assigns them) into the full [B, heads, L, d] tensor on
    every rank.  Slices are padded to the largest count for the collective."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    counts = head_counts(heads, world)
    width = max(counts)
    rank = dist.get_rank(group)
    if local.shape[1] != counts[rank]:
        raise ValueError(f"rank {rank} holds {local.shape[1]} heads, expected {counts[rank]}")
    shape = (local.shape[0], width) + tuple(local.shape[2:])
    send = torch.zeros(shape, dtype=local.dtype, device=local.device)
    send[:, :local.shape[1]] = local
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send, group=group)
    return torch.cat([p[:, :c] for p, c in zip(parts, counts)], dim=1)


def sta_forward_head_sharded(q, k, v, grid, tile, window_per_head: Sequence, scale: Optional[float] = None,
                             group=None, stream=None, gather: bool = True):
    """STA forward of raster-order [B, heads, L, d] bf16 CUDA tensors held by every
    rank of `group`: each rank computes its own heads with the CUDA path
    (``sta_forward``) and, with ``gather``, the full output is all-gathered.
    Without ``gather`` the rank's slice [B, h1 - h0, L, d] is returned.  The work
    and the result are on ``stream`` (default: the current stream)."""
    import torch.distributed as dist
    from . import _stream_context, sta_forward
    heads = int(q.shape[1])
    if len(window_per_head) != heads:
        raise ValueError("one window per head is required")
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    h0, h1 = head_range(heads, world, rank)
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    # Everything runs on `stream`: the head slices are allocated on the stream that reads
    # them, and the all-gather (which orders itself after torch's current stream) starts
    # after the local forward.
    with _stream_context(stream):
        if h1 > h0:
            local = sta_forward(q[:, h0:h1].contiguous(), k[:, h0:h1].contiguous(), v[:, h0:h1].contiguous(),
                                grid, tile, list(window_per_head[h0:h1]), scale, stream)
        else:
            local = q[:, h0:h1].new_empty((q.shape[0], 0) + tuple(q.shape[2:]))
        if not gather or world == 1:
            return local
        return gather_heads(local, heads, group)


def _world_rank(group):
    import torch.distributed as dist
    if not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def seq_to_heads(xs: Sequence, heads: int, L: int, group=None) -> List:
    """All-to-all from token shards to head shards, for several tensors in one
    collective.  Each x in ``xs`` is this rank's [B, t1 - t0, heads, d] (its
    ``token_range``); each result is [B, L, h1 - h0, d], contiguous: all tokens
    of this rank's ``head_range``."""
    import torch
    import torch.distributed as dist
    world, rank = _world_rank(group)
    n = len(xs)
    B, Lr, H, d = (int(v) for v in xs[0].shape)
    t0, t1 = token_range(L, world, rank)
    for x in xs:
        if tuple(x.shape) != (B, t1 - t0, heads, d):
            raise ValueError(f"rank {rank} holds {tuple(x.shape)}, expected {(B, t1 - t0, heads, d)}")
    if world == 1:
        return [x.contiguous() for x in xs]
    h0, h1 = head_range(heads, world, rank)
    pieces = []
    for r in range(world):
        a, b = head_range(heads, world, r)
        pieces.append(torch.stack([x[:, :, a:b] for x in xs]).reshape(-1))   # [n, B, Lr, b - a, d]
    send = torch.cat(pieces)
    in_splits = [p.numel() for p in pieces]
    counts = [b - a for a, b in (token_range(L, world, s) for s in range(world))]
    out_splits = [n * B * c * (h1 - h0) * d for c in counts]
    recv = send.new_empty(sum(out_splits))
    dist.all_to_all_single(recv, send, out_splits, in_splits, group=group)
    chunks = [c.view(n, B, cnt, h1 - h0, d) for c, cnt in zip(recv.split(out_splits), counts)]
    full = torch.cat(chunks, dim=2)                                             # [n, B, L, h1 - h0, d]
    return [full[i] for i in range(n)]


def heads_to_seq(y, heads: int, L: int, group=None):
    """Inverse of ``seq_to_heads`` for one tensor: this rank's [B, L, h1 - h0, d]
    (its heads, all tokens) to its [B, t1 - t0, heads, d] (its tokens, all
    heads)."""
    import torch
    import torch.distributed as dist
    world, rank = _world_rank(group)
    B, _, hc, d = (int(v) for v in y.shape)
    h0, h1 = head_range(heads, world, rank)
    if tuple(y.shape) != (B, L, h1 - h0, d):
        raise ValueError(f"rank {rank} holds {tuple(y.shape)}, expected {(B, L, h1 - h0, d)}")
    if world == 1:
        return y.contiguous()
    t0, t1 = token_range(L, world, rank)
    pieces = [y[:, a:b].reshape(-1) for a, b in (token_range(L, world, r) for r in range(world))]
    send = torch.cat(pieces)
    in_splits = [p.numel() for p in pieces]
    hcs = head_counts(heads, world)
    out_splits = [B * (t1 - t0) * c * d for c in hcs]
    recv = send.new_empty(sum(out_splits))
    dist.all_to_all_single(recv, send, out_splits, in_splits, group=group)
    chunks = [c.view(B, t1 - t0, hc_s, d) for c, hc_s in zip(recv.split(out_splits), hcs)]
    return torch.cat(chunks, dim=2)


def sta_forward_sequence_sharded(q, k, v, grid, tile, window_per_head: Sequence, scale: Optional[float] = None,
                                 group=None):
    """STA forward of sequence-sharded token-major tensors: q, k, v are this rank's
    [B, t1 - t0, heads, d] bf16 CUDA tensors (its ``token_range`` of the L = T*H*W
    raster-order tokens); returns the output for the same tokens,
    [B, t1 - t0, heads, d].  The grid must be a tile multiple."""
    import torch
    from . import sta_forward_tokens
    heads = int(q.shape[2])
    L = int(grid[0]) * int(grid[1]) * int(grid[2])
    if len(window_per_head) != heads:
        raise ValueError("one window per head is required")
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    world, rank = _world_rank(group)
    h0, h1 = head_range(heads, world, rank)
    qh, kh, vh = seq_to_heads([q, k, v], heads, L, group)
    if h1 > h0:
        oh = sta_forward_tokens(qh, kh, vh, grid, tile, list(window_per_head[h0:h1]), scale)
    else:
        oh = torch.empty((q.shape[0], L, 0, q.shape[3]), dtype=q.dtype, device=q.device)
    return heads_to_seq(oh, heads, L, group)
