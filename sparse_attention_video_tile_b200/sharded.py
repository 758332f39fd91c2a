"""Head-sharded STA forward over several GPUs (one process per GPU).

(batch, head) pairs of Sliding Tile Attention are independent and each head has
its own window, so heads split across ranks with no exchange inside attention:
every rank runs the CUDA path on its contiguous range of heads.  The only
collective is the all-gather that gives every rank the full output afterwards
(NCCL over NVLink on B200; any torch.distributed backend works for the host
logic).

This module holds host logic only: the head partition, the call into the CUDA
path for the local heads, and the gather.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple


def head_range(heads: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous range [h0, h1) of the heads owned by `rank`: the first
    heads % world ranks take one head more than the others."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if heads < 0:
        raise ValueError("heads must be non-negative")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


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
    Without ``gather`` the rank's slice [B, h1 - h0, L, d] is returned."""
    import torch.distributed as dist
    from . import sta_forward
    heads = int(q.shape[1])
    if len(window_per_head) != heads:
        raise ValueError("one window per head is required")
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    h0, h1 = head_range(heads, world, rank)
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    if h1 > h0:
        local = sta_forward(q[:, h0:h1].contiguous(), k[:, h0:h1].contiguous(), v[:, h0:h1].contiguous(),
                            grid, tile, list(window_per_head[h0:h1]), scale, stream)
    else:
        local = q[:, h0:h1].new_empty((q.shape[0], 0) + tuple(q.shape[2:]))
    if not gather or world == 1:
        return local
    return gather_heads(local, heads, group)
