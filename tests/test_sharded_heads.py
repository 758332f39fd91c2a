"""Host logic of the head-sharded forward (sparse_attention_video_tile_b200.sharded)
on CPU: the head partition, and the all-gather of per-rank head slices with two
gloo ranks.  The attention itself runs only on the GPU (GPU tests); here each rank
fills its slice with values that identify (batch, head, row, column)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_video_tile_b200.sharded import gather_heads, head_counts, head_range


@pytest.mark.parametrize("heads,world", [(24, 1), (24, 2), (24, 8), (7, 3), (3, 4), (0, 2), (25, 8)])
def test_head_ranges_partition_the_heads(heads, world):
    ranges = [head_range(heads, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == heads
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0                        # contiguous, in rank order, disjoint
    counts = head_counts(heads, world)
    assert sum(counts) == heads and max(counts) - min(counts) <= 1
    with pytest.raises(ValueError):
        head_range(heads, world, world)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full_reference(B, heads, L, d):
    b, h, l, c = torch.meshgrid(torch.arange(B), torch.arange(heads), torch.arange(L), torch.arange(d), indexing="ij")
    return (1000 * b + 100 * h + 10 * l + c).to(torch.float32)


def _rank_main(rank, world, port, heads, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, L, d = 2, 3, 4
        h0, h1 = head_range(heads, world, rank)
        local = _full_reference(B, heads, L, d)[:, h0:h1].contiguous()
        full = gather_heads(local, heads)
        results[rank] = torch.equal(full, _full_reference(B, heads, L, d))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("heads", [24, 5])
def test_gather_reassembles_every_rank_full_output(heads):
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), heads, results), nprocs=world, join=True,
                           start_method="spawn")
        assert dict(results) == {0: True, 1: True}


@pytest.mark.gpu
def test_head_slices_on_one_gpu_equal_the_full_forward():
    """What each rank computes (its contiguous heads through the CUDA path), put
    side by side, is bit-identical to the full forward: heads are independent."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import workloads as W
    import sparse_attention_video_tile_b200 as sta
    from sparse_attention_video_tile_b200.build import build
    from sparse_attention_video_tile_b200.sharded import sta_forward_head_sharded
    build()
    cfg = W.custom_config("shard", 1, 5, 128, (12, 24, 40), (6, 8, 8), [(1, 3, 3), (3, 3, 3), (1, 1, 1), (3, 5, 5), (1, 3, 3)])
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, 9))
    full = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    alone = sta_forward_head_sharded(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale)   # one process
    parts = []
    for r in range(2):
        h0, h1 = head_range(cfg.heads, 2, r)
        parts.append(sta.sta_forward(q[:, h0:h1].contiguous(), k[:, h0:h1].contiguous(), v[:, h0:h1].contiguous(),
                                     cfg.grid, cfg.tile, cfg.windows[h0:h1], cfg.scale))
    torch.cuda.synchronize()
    assert torch.equal(alone, full)
    assert torch.equal(torch.cat(parts, dim=1), full)
