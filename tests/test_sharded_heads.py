"""Host logic of the sharded forwards (sparse_attention_video_tile_b200.sharded)
on CPU: the head and token partitions, the all-gather of per-rank head slices,
and the two all-to-alls of the sequence-sharded forward, with gloo ranks.  The
attention itself runs only on the GPU (GPU tests); here each rank fills its
slice with values that identify (batch, head, row, column)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_video_tile_b200.sharded import (gather_heads, head_counts, head_range, heads_to_seq,
                                                     seq_to_heads, token_range)


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


def _a2a_main(rank, world, port, heads, L, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, d = 2, 4
        full = _full_reference(B, heads, L, d).transpose(1, 2).contiguous()     # token-major [B, L, heads, d]
        t0, t1 = token_range(L, world, rank)
        h0, h1 = head_range(heads, world, rank)
        local = full[:, t0:t1].contiguous()
        twice = 2 * local
        got_q, got_k = seq_to_heads([local, twice], heads, L)                  # one collective for both
        ok = torch.equal(got_q, full[:, :, h0:h1]) and torch.equal(got_k, 2 * full[:, :, h0:h1])
        ok = ok and got_q.is_contiguous() and got_k.is_contiguous()
        # a per-head stand-in for attention, then back to this rank's tokens
        head_ids = torch.arange(h0, h1, dtype=torch.float32).view(1, 1, -1, 1)
        back = heads_to_seq(got_q * (head_ids + 1), heads, L)
        want = local * (torch.arange(heads, dtype=torch.float32).view(1, 1, -1, 1) + 1)
        results[rank] = bool(ok and torch.equal(back, want))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("heads,L,world", [(24, 64, 2), (5, 7, 2), (1, 9, 2), (4, 10, 3)])
def test_sequence_shards_exchange_to_head_shards_and_back(heads, L, world):
    """Uneven token and head splits, and a rank with no heads (1 head, 2 ranks)."""
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_a2a_main, args=(world, _free_port(), heads, L, results), nprocs=world, join=True,
                           start_method="spawn")
        assert dict(results) == {r: True for r in range(world)}


def test_token_ranges_partition_the_tokens():
    for L, world in ((115200, 8), (7, 3), (2, 4)):
        ranges = [token_range(L, world, r) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == L
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))


@pytest.mark.gpu
def test_sequence_sharded_single_rank_equals_token_major_forward():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import workloads as W
    import sparse_attention_video_tile_b200 as sta
    from sparse_attention_video_tile_b200.build import build
    from sparse_attention_video_tile_b200.sharded import sta_forward_sequence_sharded
    build()
    cfg = W.custom_config("seq_shard", 1, 3, 128, (12, 24, 40), (6, 8, 8), [(1, 3, 3), (3, 3, 3), (1, 1, 1)])
    import numpy as np
    import oracle.sta_oracle as O
    q0, k0, v0 = W.make_qkv(cfg, 10)
    q, k, v = (x.cuda().transpose(1, 2).contiguous() for x in (q0, k0, v0))
    want = sta.sta_forward_tokens(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    got = sta_forward_sequence_sharded(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    out = got.float().cpu().numpy().astype(np.float64)        # [B, L, heads, d]
    for h in range(cfg.heads):
        ref = O.sta_attention_head(q0[0, h].double().numpy(), k0[0, h].double().numpy(), v0[0, h].double().numpy(),
                                   cfg.grid, cfg.tile, cfg.windows[h], cfg.scale)
        assert np.abs(out[0, :, h] - ref).max() <= 1e-2
        assert np.linalg.norm(out[0, :, h] - ref) / np.linalg.norm(ref) <= 5e-3


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


def _gpu_rank_main(rank, world, port, results):
    """One rank of the head-sharded forward on the one GPU of the run: it computes
    its own heads (no collective: gather=False) and checks them against the oracle."""
    import numpy as np
    import oracle.sta_oracle as O
    import workloads as W
    import sparse_attention_video_tile_b200 as sta
    from sparse_attention_video_tile_b200.sharded import sta_forward_head_sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        sta.load_library()
        cfg = W.custom_config("shard_oracle", 1, 5, 128, (12, 24, 40), (6, 8, 8),
                              [(1, 3, 3), (3, 3, 3), (1, 1, 1), (3, 5, 5), (2, 3, 5)])
        q, k, v = W.make_qkv(cfg, 9)
        part = sta_forward_head_sharded(q.cuda(), k.cuda(), v.cuda(), cfg.grid, cfg.tile, cfg.windows, cfg.scale,
                                        gather=False)
        torch.cuda.synchronize()
        h0, h1 = head_range(cfg.heads, world, rank)
        assert part.shape == (1, h1 - h0, cfg.L, cfg.d), part.shape
        assert sta.sta_check_device_status() == sta.STA_OK
        got = part.float().cpu().numpy().astype(np.float64)
        worst = (0.0, 0.0)
        for i, h in enumerate(range(h0, h1)):
            want = O.sta_attention_head(q[0, h].double().numpy(), k[0, h].double().numpy(), v[0, h].double().numpy(),
                                        cfg.grid, cfg.tile, cfg.windows[h], cfg.scale)
            err = float(np.abs(got[0, i] - want).max())
            rel = float(np.linalg.norm(got[0, i] - want) / np.linalg.norm(want))
            worst = (max(worst[0], err), max(worst[1], rel))
        results[rank] = (h0, h1, worst[0], worst[1])
    except Exception as e:  # reported to the parent
        results[rank] = repr(e)
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_head_sharded_slices_match_the_oracle():
    """Each of two ranks computes its contiguous heads (per-head windows) through
    the CUDA path; every row of every head is compared with the oracle.  The ranks
    share the run's one GPU; their kernels are independent (no collective)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_video_tile_b200.build import build
    build()
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_gpu_rank_main, args=(world, _free_port(), results), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(results)
    covered = []
    for r in range(world):
        assert not isinstance(res[r], str), f"rank {r}: {res[r]}"
        h0, h1, err, rel = res[r]
        covered += list(range(h0, h1))
        assert err <= 1e-2 and rel <= 5e-3, f"rank {r} heads [{h0}, {h1}): max abs {err:.3e}, rel {rel:.3e}"
    assert covered == list(range(5))
