"""Host logic of bench.py's multi-GPU runs, on CPU with two gloo ranks.

With N GPUs the bench runs N independent replicas (the path has no exchange
step): each rank times its own replica, the job's time is the slowest rank's
(a max over ranks), the job's value counts the work of all ranks, and the
reference arm runs on rank 0 only.  The collective here is the same call the
bench makes, on the gloo backend instead of NCCL.
"""
import contextlib
import io
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank step times: the slowest rank decides
        ms = [12.5, 14.0][rank]
        job_ms = bench.max_over_ranks(ms, torch.device("cpu"))
        value = bench.job_tflops(world, 1.0e13, job_ms)
        # the reference arm prints on rank 0 only; other ranks return 0 at once
        args = type("A", (), {"ref_rows": 1, "warmup": 3, "steps": 1, "gpus": world})()
        buf = io.StringIO()
        rc = None
        if rank == 1:
            with contextlib.redirect_stdout(buf):
                rc = bench.run_reference(args, None)
        results[rank] = (job_ms, value, rc, buf.getvalue())
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank_and_count_all_work():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(results)
    for rank in range(world):
        job_ms, value, _, _ = res[rank]
        assert job_ms == 14.0
        assert value == pytest.approx(2 * 1.0e13 / 14.0e-3 / 1e12)
    _, _, rc, out = res[1]
    assert rc == 0 and out == ""


def test_single_process_is_the_identity():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25
    assert bench.job_tflops(1, 2.0e12, 1000.0) == pytest.approx(2.0)  # 2e12 FLOP in one second
