"""The checked build (libsta_checked.so, compiled with STA_DEVICE_CHECKS=1) on the GPU.

It tests, inside the forward kernel, every index taken from the work schedule
(work items, key-block rows, mask ids) and every computed output row before it
is used, and reports a failed check as STA_ERR_BOUNDS after skipping the access.
This stands in for a memory checker, which is not available here.  The checks
must not change the arithmetic: the checked library's outputs equal the
production library's bit for bit.  A test-only switch of the checked build
plants a key-block row far past the tensor (a tensor-map load there would read
zeros, not fault): the kernel must catch it, and the context must stay usable.
"""
import ctypes
import os
import subprocess
import sys

import pytest
import torch

import workloads as W
import sparse_attention_video_tile_b200 as sta

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
STA_ERR_BOUNDS = 12


def _load(path):
    lib = ctypes.CDLL(path)
    P, I32, I64, D3, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, sta.sta_dim3, ctypes.c_float
    for name in ("sta_attention_fwd", "sta_attention_fwd_raster", "sta_attention_fwd_mixed"):
        fn = getattr(lib, name)
        fn.restype = ctypes.c_int
        fn.argtypes = [P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), F, P]
    lib.sta_attention_fwd_lse.restype = ctypes.c_int
    lib.sta_attention_fwd_lse.argtypes = [P, P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), F, P]
    lib.sta_attention_bwd.restype = ctypes.c_int
    lib.sta_attention_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I32, I32, I32, D3, D3, ctypes.POINTER(D3), F, P]
    lib.sta_check_device_status.restype = ctypes.c_int
    lib.sta_check_device_status.argtypes = [P]
    return lib


def _backward(lib, cfg, q, k, v, do):
    """Forward with log-sum-exp and backward through `lib` on tiled tensors."""
    B, Hn, L, d = q.shape
    s = torch.cuda.current_stream().cuda_stream
    out = torch.empty_like(q)
    lse = torch.empty((B, Hn, L), device=q.device, dtype=torch.float32)
    g3, t3, w = sta._d3(cfg.grid), sta._d3(cfg.tile), sta._windows(cfg.windows)
    assert lib.sta_attention_fwd_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hn, d,
                                     g3, t3, w, ctypes.c_float(cfg.scale), s) == 0
    grads = [torch.full_like(q, float("nan")) for _ in range(3)]
    assert lib.sta_attention_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), do.data_ptr(), lse.data_ptr(),
                                 *(g.data_ptr() for g in grads), B, Hn, d, g3, t3, w, ctypes.c_float(cfg.scale), s) == 0
    return grads


@pytest.fixture(scope="module")
def checked():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_video_tile_b200.build import LIB_CHECKED, build
    build()
    sta.load_library()
    torch.cuda.set_device(0)
    return _load(LIB_CHECKED)


def _call(lib, name, q, k, v, out, cfg):
    B, Hn, _, d = q.shape
    return getattr(lib, name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hn, d, sta._d3(cfg.grid),
                              sta._d3(cfg.tile), sta._windows(cfg.windows), ctypes.c_float(cfg.scale),
                              torch.cuda.current_stream().cuda_stream)


CASES = [
    ("tiled", W.CONFIGS["tiny"]),                  # masked path (32-token tiles), d = 64
    ("tiled", W.CONFIGS["small"]),
    ("tiled", W.custom_config("batch2", 2, 3, 128, (4, 16, 24), (2, 8, 8), [(1, 1, 1), (3, 3, 3), (1, 2, 3)])),
    ("raster", W.custom_config("pad_perhead", 1, 3, 128, (13, 17, 20), (6, 8, 8), [(1, 3, 3), (3, 5, 5), (5, 6, 10)])),
    ("mixed", W.custom_config("pad_image", 2, 2, 128, (1, 30, 45), (1, 8, 16), [(1, 5, 3), (1, 3, 3)])),
    ("mixed", W.CONFIGS["image2d"]),
]


@pytest.mark.parametrize("path,cfg", CASES, ids=lambda x: x if isinstance(x, str) else x.name)
def test_checked_build_passes_and_matches_production(checked, path, cfg):
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, 5))
    got = torch.full_like(q, float("nan"))
    if path == "tiled":
        qt, kt, vt = (torch.empty_like(x) for x in (q, k, v))
        for a, b in ((q, qt), (k, kt), (v, vt)):
            sta.sta_tile_reorder(a, b, cfg.grid, cfg.tile)
        want = torch.empty_like(q)
        sta.sta_attention_fwd(qt, kt, vt, want, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
        assert _call(checked, "sta_attention_fwd", qt, kt, vt, got, cfg) == 0
    elif path == "raster":
        want = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale, path="fused")
        assert _call(checked, "sta_attention_fwd_raster", q, k, v, got, cfg) == 0
    else:
        kp, vp = (torch.empty((cfg.batch, cfg.heads, sta.padded_rows(cfg.grid, cfg.tile), cfg.d), dtype=q.dtype,
                              device=q.device) for _ in range(2))
        sta.sta_tile_reorder_padded(k, kp, cfg.grid, cfg.tile)
        sta.sta_tile_reorder_padded(v, vp, cfg.grid, cfg.tile)
        want = torch.empty_like(q)
        sta.sta_attention_fwd_mixed(q, kp, vp, want, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
        assert _call(checked, "sta_attention_fwd_mixed", q, kp, vp, got, cfg) == 0
    assert checked.sta_check_device_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    assert torch.equal(got, want)


def test_checked_build_backward_matches_production(checked):
    cfg = W.custom_config("bwd_checked", 2, 3, 64, (4, 16, 24), (2, 8, 8), [(1, 1, 1), (3, 3, 3), (1, 2, 3)])
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, 5))
    do = W.make_qkv(cfg, 105)[0].cuda()
    got = _backward(checked, cfg, q, k, v, do)
    assert checked.sta_check_device_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    want = _backward(sta.load_library(), cfg, q, k, v, do)
    torch.cuda.synchronize()
    for a, b in zip(got, want):
        assert torch.equal(a, b)


PLANT = r"""
import ctypes, os, sys, torch
sys.path.insert(0, ROOT)
sys.path.insert(0, HERE)
import workloads as W
import sparse_attention_video_tile_b200 as sta
from sparse_attention_video_tile_b200.build import LIB_CHECKED
from test_gpu_device_checks import _load, _call, _backward
sta.load_library()
lib = _load(LIB_CHECKED)
s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
cfg = W.custom_config("plant", 1, 2, 128, (6, 24, 32), (6, 8, 8), [(1, 3, 3), (1, 1, 1)])
q, k, v = (x.cuda() for x in W.make_qkv(cfg, 1))
out = torch.empty_like(q)
assert _call(lib, "sta_attention_fwd", q, k, v, out, cfg) == 0     # schedule built with the planted row
print("status", lib.sta_check_device_status(s))
cfgb = W.custom_config("plant_bwd", 1, 2, 128, (6, 24, 24), (6, 8, 8), [(1, 3, 3), (1, 1, 1)])
q, k, v = (x.cuda() for x in W.make_qkv(cfgb, 2))
do = W.make_qkv(cfgb, 3)[0].cuda()
_backward(lib, cfgb, q, k, v, do)             # the forward and the transposed schedules carry the planted row
print("bwd", lib.sta_check_device_status(s))
os.environ.pop("STA_CHECKS_PLANT_BAD_ROW")
cfg2 = W.custom_config("clean", 1, 2, 128, (6, 24, 40), (6, 8, 8), [(1, 3, 3), (1, 1, 1)])
q, k, v = (x.cuda() for x in W.make_qkv(cfg2, 1))
out = torch.empty_like(q)
assert _call(lib, "sta_attention_fwd", q, k, v, out, cfg2) == 0    # a new configuration: a clean schedule
print("after", lib.sta_check_device_status(s), bool(torch.isfinite(out.float()).all()))
"""


def test_checked_build_catches_a_planted_bad_row(checked):
    env = dict(os.environ, STA_CHECKS_PLANT_BAD_ROW="1")
    code = PLANT.replace("ROOT", repr(ROOT)).replace("HERE", repr(HERE))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = dict(l.split(" ", 1) for l in r.stdout.strip().splitlines() if " " in l)
    assert lines["status"].strip() == str(STA_ERR_BOUNDS), r.stdout
    assert lines["bwd"].strip() == str(STA_ERR_BOUNDS), r.stdout
    assert lines["after"].strip() == "0 True", r.stdout
