"""sta_attention_fwd_noalloc against sta_attention_fwd, through the C ABI.

The no-alloc entry point serves callers that cannot let a library call
cudaMalloc (code inside a memory pool or arena it must not bypass, processes
that reserve all device memory up front, allocators that must account for every
device allocation).  It keeps the attention kernel's scratch (status word and
work schedule) in a fixed static device array instead.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test.  It must pass on its own in a fresh
process (the first call sets up the array's device address) and after the other
tests.

A kernel of this entry point that gives up on a bounded wait records it in the
array's status word; sta_check_device_status reads and clears that word, and
sta_selftest_bounded_wait runs a wait out through it.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
import sparse_attention_video_tile_b200 as sta

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_FRO = 5e-3
STA_ERR_SCRATCH = 11


@pytest.fixture(scope="module")
def noalloc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_video_tile_b200.build import build
    build()
    lib = sta.load_library()
    torch.cuda.set_device(0)
    fn = lib.sta_attention_fwd_noalloc
    P, I32, D3 = ctypes.c_void_p, ctypes.c_int32, sta.sta_dim3
    fn.restype = ctypes.c_int
    fn.argtypes = [P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), ctypes.c_float, P]
    return fn


def _call(fn, q, k, v, out, cfg):
    B, Hn, L, d = q.shape
    return fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hn, d, sta._d3(cfg.grid),
              sta._d3(cfg.tile), sta._windows(cfg.windows), ctypes.c_float(cfg.scale),
              torch.cuda.current_stream().cuda_stream)


def _check_against_allocating_entry(fn, cfg, seed):
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, seed))
    qt, kt, vt = (torch.empty_like(x) for x in (q, k, v))
    for src, dst in ((q, qt), (k, kt), (v, vt)):
        sta.sta_tile_reorder(src, dst, cfg.grid, cfg.tile)
    ref = torch.empty_like(qt)
    sta.sta_attention_fwd(qt, kt, vt, ref, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    got = torch.full_like(qt, float("nan"))
    assert _call(fn, qt, kt, vt, got, cfg) == 0
    torch.cuda.synchronize()
    # the call's status word (and the allocating path's) report no expired wait
    assert sta.sta_check_device_status() == sta.STA_OK
    a = got.float().cpu().numpy().astype(np.float64)
    b = ref.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(a))
    assert np.abs(a - b).max() <= MAX_ABS
    assert np.linalg.norm(a - b) / np.linalg.norm(b) <= REL_FRO


def test_noalloc_matches_allocating_entry_on_consecutive_calls(noalloc):
    small = W.CONFIGS["small"]
    other = W.custom_config("batch2", 2, 3, 128, (4, 16, 24), (2, 8, 8), [(1, 1, 1), (3, 3, 3), (1, 2, 3)])
    _check_against_allocating_entry(noalloc, small, 7)    # first call: set-up and upload
    _check_against_allocating_entry(noalloc, other, 8)    # second call: another schedule replaces it
    _check_against_allocating_entry(noalloc, small, 9)    # back to the first configuration
    _check_against_allocating_entry(noalloc, W.CONFIGS["tiny"], 10)  # masked path, d = 64


def test_noalloc_rejects_schedule_larger_than_scratch(noalloc):
    # One dense head on a 16x6x10 tile grid: about 11 MB of key-block lists, more than
    # the 4 MiB scratch.  The call must fail before touching the (never dereferenced)
    # tensor pointers.
    cfg = W.custom_config("huge", 1, 1, 128, (96, 48, 80), (6, 8, 8), [(16, 6, 10)])
    span = 1 << 40
    st = noalloc(1 * span, 2 * span, 3 * span, 4 * span, 1, 1, 128, sta._d3(cfg.grid), sta._d3(cfg.tile),
                 sta._windows(cfg.windows), ctypes.c_float(cfg.scale), torch.cuda.current_stream().cuda_stream)
    assert st == STA_ERR_SCRATCH
    assert sta.sta_status_str(st) == "STA_ERR_SCRATCH"


def test_noalloc_timeouts_are_reported_and_cleared(noalloc):
    # After a good call its status word is clear ...
    _check_against_allocating_entry(noalloc, W.CONFIGS["tiny"], 11)
    # ... a wait run out through every status word of the device (the no-alloc
    # array's among them, now that it is set up) is reported ...
    assert sta.sta_selftest_bounded_wait(20_000_000) == sta.STA_ERR_TIMEOUT
    # ... and the check after it finds every word cleared.
    assert sta.sta_check_device_status() == sta.STA_OK
    # The next call still computes correctly and leaves its word clear.
    _check_against_allocating_entry(noalloc, W.CONFIGS["small"], 12)


def test_noalloc_after_shutdown_sets_up_again(noalloc):
    _check_against_allocating_entry(noalloc, W.CONFIGS["small"], 13)
    sta.sta_shutdown()
    # the same configuration again: the set-up and the upload are redone
    _check_against_allocating_entry(noalloc, W.CONFIGS["small"], 14)
    _check_against_allocating_entry(noalloc, W.CONFIGS["small"], 15)
