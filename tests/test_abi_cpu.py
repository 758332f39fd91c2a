"""C-ABI checks that need no GPU: exported symbols, host-only entry points
against the oracle, and argument validation (which returns before any device
call).  With valid arguments on a machine without a GPU the product path must
fail loudly (a CUDA or architecture error), never fall back to the CPU.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle.sta_oracle as O
import workloads as W
from workloads import CONFIGS

import sparse_attention_video_tile_b200 as sta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    txt = open(os.path.join(ROOT, "include", "sta.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(sta_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_video_tile_b200.build import build
    build()
    return sta.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


def test_header_is_plain_c_and_matches_the_library(lib, tmp_path):
    """tests/c/abi_from_c.c binds every entry point to a pointer of its spelled-out
    type (C99, -Werror), links against libsta.so and calls the host entry points."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    pkg = os.path.dirname(sta.LIB_PATH)
    exe = str(tmp_path / "abi_from_c")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_from_c.c"), "-o", exe, "-L", pkg, "-l:libsta.so",
           "-Wl,-rpath," + pkg]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    env = dict(os.environ)
    import torch   # its bundled CUDA runtime is the one libsta.so resolves at run time
    env["LD_LIBRARY_PATH"] = os.pathsep.join(
        [os.path.join(os.path.dirname(torch.__file__), "lib")] +
        [p for p in (os.path.join(os.path.dirname(os.path.dirname(torch.__file__)), "nvidia", "cuda_runtime", "lib"),)
         if os.path.isdir(p)] + [env.get("LD_LIBRARY_PATH", "")])
    out = subprocess.run([exe], check=True, capture_output=True, text=True, env=env).stdout.splitlines()
    got_map = np.array([int(x) for x in out[0].split()[1:]], dtype=np.int64)
    assert np.array_equal(got_map, O.tiled_of_raster((4, 8, 8), (2, 4, 4)))
    assert int(out[1].split()[1]) == O.attended_pairs(1, (4, 8, 8), (2, 4, 4), [(1, 1, 1), (3, 3, 3)])
    assert out[2].split()[1:] == ["STA_OK", "STA_ERR_SHAPE"]
    assert out[3].split()[1] == "STA_ERR_NULL"


def test_status_strings(lib):
    for code, name in sta.STATUS_NAMES.items():
        assert sta.sta_status_str(code) == name


@pytest.mark.parametrize("grid,tile", [((2, 2, 4), (1, 2, 2)), ((4, 8, 8), (2, 4, 4)), ((12, 24, 40), (6, 8, 8)),
                                       ((30, 48, 80), (6, 8, 8)), ((1, 128, 128), (1, 8, 16)),
                                       ((48, 48, 80), (6, 8, 8)), ((3, 10, 10), (1, 5, 5))])
def test_index_map_bit_exact_vs_oracle(lib, grid, tile):
    got = sta.sta_tile_index_map(grid, tile)
    want = O.tiled_of_raster(grid, tile)
    assert got.dtype == np.int32
    assert np.array_equal(got.astype(np.int64), want)


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_attended_pairs_vs_oracle(lib, name):
    c = CONFIGS[name]
    assert sta.sta_attended_pairs(c.batch, c.heads, c.grid, c.tile, c.windows) == \
        O.attended_pairs(c.batch, c.grid, c.tile, c.windows)


def _call_reorder(lib, src, dst, bh=1, d=128, grid=(4, 8, 8), tile=(2, 4, 4)):
    return lib.sta_tile_reorder(src, dst, bh, d, sta._d3(grid), sta._d3(tile), None)


def _call_attn(lib, q=0x10000, k=0x20000, v=0x30000, out=0x40000, batch=1, heads=2, d=64,
               grid=(4, 8, 8), tile=(2, 4, 4), windows=((1, 1, 1), (3, 3, 3)), scale=0.125):
    return lib.sta_attention_fwd(q, k, v, out, batch, heads, d, sta._d3(grid), sta._d3(tile),
                                 sta._windows(windows), ctypes.c_float(scale), None)


def test_validation_codes(lib):
    A, B = 0x100000, 0x200000   # fake, never dereferenced: validation fails first
    assert _call_reorder(lib, None, B) == 1
    assert _call_reorder(lib, A + 2, B) == 2
    assert _call_reorder(lib, A, A) == 3
    assert _call_reorder(lib, A, A + 1024) == 3                      # overlapping ranges
    assert _call_reorder(lib, A, B, grid=(4, 8, 9)) == 4
    assert _call_reorder(lib, A, B, grid=(0, 8, 8)) == 4
    assert _call_reorder(lib, A, B, d=96) == 6
    assert lib.sta_tile_unorder(A, B, 1, 128, sta._d3((4, 8, 9)), sta._d3((2, 4, 4)), None) == 4
    assert _call_attn(lib, q=None) == 1
    assert _call_attn(lib, out=0x40008) == 2
    assert _call_attn(lib, out=0x10000) == 3
    assert _call_attn(lib, d=80) == 6
    assert _call_attn(lib, tile=(3, 4, 4)) == 4
    assert _call_attn(lib, windows=((1, 0, 1), (3, 3, 3))) == 5
    assert _call_attn(lib, scale=0.0) == 10
    assert _call_attn(lib, scale=float("nan")) == 10
    assert _call_attn(lib, batch=0) == 10
    assert lib.sta_tile_index_map(sta._d3((4, 8, 8)), sta._d3((2, 4, 4)), None) == 1
    assert lib.sta_attended_pairs(1, 1, sta._d3((4, 8, 8)), sta._d3((3, 4, 4)), sta._windows([(1, 1, 1)])) == -1


def _call_tokens(lib, src, dst, batch=1, heads=2, d=128, grid=(4, 8, 8), tile=(2, 4, 4), unorder=False):
    fn = lib.sta_tile_unorder_tokens if unorder else lib.sta_tile_reorder_tokens
    return fn(src, dst, batch, heads, d, sta._d3(grid), sta._d3(tile), None)


def test_token_major_reorder_validation_codes(lib):
    # fake pointers, never dereferenced; one tensor is 2 x 256 x 128 bf16 = 128 KB
    A, B = 0x100000, 0x200000
    for unorder in (False, True):
        assert _call_tokens(lib, None, B, unorder=unorder) == 1
        assert _call_tokens(lib, A, 0, unorder=unorder) == 1
        assert _call_tokens(lib, A + 8, B, unorder=unorder) == 2
        assert _call_tokens(lib, A, A + 64 * 1024, unorder=unorder) == 3      # the second half of src
        assert _call_tokens(lib, A, B, grid=(4, 8, 9), unorder=unorder) == 4
        assert _call_tokens(lib, A, B, d=32, unorder=unorder) == 6
        assert _call_tokens(lib, A, B, batch=-1, unorder=unorder) == 10
        assert _call_tokens(lib, A, B, heads=-2, unorder=unorder) == 10


def _call_bwd(lib, base=0x1000000, lse=0x9000000, batch=1, heads=1, d=128, grid=(6, 8, 16), tile=(6, 8, 8),
              windows=((1, 1, 1),), scale=0.1, **ptrs):
    # q, k, v, out, dout, dq, dk, dv spaced 1 MB apart (each [1, 1, 768, 128] bf16 = 192 KB)
    names = ("q", "k", "v", "out", "dout", "dq", "dk", "dv")
    p = {n: base + i * (1 << 20) for i, n in enumerate(names)}
    p.update(ptrs)
    return lib.sta_attention_bwd(p["q"], p["k"], p["v"], p["out"], p["dout"], lse, p["dq"], p["dk"], p["dv"],
                                 batch, heads, d, sta._d3(grid), sta._d3(tile), sta._windows(windows),
                                 ctypes.c_float(scale), None)


def test_backward_validation_codes(lib):
    # fake pointers, never dereferenced: validation fails before the device is touched
    assert _call_bwd(lib, q=None) == 1
    assert _call_bwd(lib, lse=None) == 1
    assert _call_bwd(lib, dk=0x1000000 + 5 * (1 << 20) + 8) == 2
    assert _call_bwd(lib, lse=0x9000004) == 2
    assert _call_bwd(lib, d=96) == 6
    assert _call_bwd(lib, grid=(4, 8, 8), tile=(2, 4, 4)) == 4         # 32-token tiles: not a multiple of 128
    assert _call_bwd(lib, grid=(6, 8, 17)) == 4
    assert _call_bwd(lib, windows=((0, 1, 1),)) == 5
    assert _call_bwd(lib, scale=-1.0) == 10
    assert _call_bwd(lib, dq=0x1000000) == 3                            # dq over q
    assert _call_bwd(lib, dv=0x1000000 + 5 * (1 << 20)) == 3           # dv over dq
    assert _call_bwd(lib, lse=0x1000000 + 6 * (1 << 20)) == 3          # lse inside dk


def test_no_cpu_fallback_without_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # valid arguments: the library must report a CUDA/architecture error, not compute on the host
    assert _call_reorder(lib, 0x100000, 0x200000) in (7, 8)
    assert _call_tokens(lib, 0x100000, 0x200000) in (7, 8)
    assert _call_tokens(lib, 0x100000, 0x200000, unorder=True) in (7, 8)
    # the overlap check covers batch * heads * L * d elements: disjoint when that is smaller
    assert _call_tokens(lib, 0x100000, 0x100000 + 64 * 1024, heads=1) in (7, 8)
    assert _call_attn(lib) in (7, 8)
    assert _call_bwd(lib) in (7, 8)
    assert _call_host(lib) in (7, 8)


def test_python_paths_refuse_cpu_tensors(lib):
    """The binding hands device pointers to the library and nothing else: host
    tensors are refused before any call, on every path."""
    import torch
    from sparse_attention_video_tile_b200.autograd import sta_attention
    cfg = W.custom_config("cpu_refusal", 1, 2, 64, (2, 8, 16), (2, 8, 8), [(1, 1, 1), (1, 1, 2)])
    q, k, v = W.make_qkv(cfg, 0)
    tq = q.transpose(1, 2).contiguous()
    with pytest.raises(ValueError, match="CUDA"):
        sta.sta_forward_tokens(tq, tq, tq, cfg.grid, cfg.tile, cfg.windows)
    with pytest.raises(ValueError, match="CUDA"):
        sta_attention(q, k, v, cfg.grid, cfg.tile, cfg.windows)
    with pytest.raises(ValueError, match="does not match"):
        sta.sta_tile_reorder_tokens(tq, torch.empty_like(tq), cfg.grid, cfg.tile)


SCHEDULE_CASES = [
    ("small", None),
    ("b2_perhead", W.custom_config("b2_perhead", 2, 3, 64, (4, 16, 24), (2, 8, 8), [(1, 1, 1), (3, 3, 3), (1, 2, 3)])),
    ("image", W.custom_config("image", 1, 2, 128, (1, 32, 48), (1, 8, 16), [(1, 3, 3), (1, 4, 2)])),
    ("even", W.custom_config("even", 1, 1, 128, (6, 32, 32), (2, 8, 8), [(2, 2, 4)])),
]


@pytest.mark.parametrize("name,cfg", SCHEDULE_CASES, ids=[c[0] for c in SCHEDULE_CASES])
def test_schedules_cover_exactly_the_window_blocks(lib, name, cfg):
    """Both work schedules (forward: query blocks with their key blocks; backward:
    key blocks with their query blocks) hold exactly the block pairs whose tiles the
    oracle's window rule connects, each once."""
    cfg = cfg or W.CONFIGS[name]
    tiled = O.tiled_of_raster(cfg.grid, cfg.tile)
    raster_of_tiled = np.empty_like(tiled)
    raster_of_tiled[tiled] = np.arange(tiled.size)
    coords = O.raster_coords(cfg.grid)
    nblk = cfg.L // 128
    rep = coords[raster_of_tiled[np.arange(nblk) * 128]]       # one token of each 128-row block
    want = set()
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            m = O.sta_mask(rep, rep, cfg.grid, cfg.tile, cfg.windows[h])
            qi, ki = np.nonzero(m)
            want.update(zip([b * cfg.heads + h] * len(qi), (qi * 128).tolist(), (ki * 128).tolist()))
    for transposed in (False, True):
        got = sta.sta_schedule_block_pairs(cfg.batch, cfg.heads, cfg.grid, cfg.tile, cfg.windows, transposed)
        triples = list(map(tuple, got.tolist()))
        assert len(triples) == len(set(triples)), "a block pair appears twice"
        assert set(triples) == want
        assert len(triples) * 128 * 128 == O.attended_pairs(cfg.batch, cfg.grid, cfg.tile, cfg.windows)


def test_schedule_pairs_reject_small_tiles(lib):
    assert lib.sta_schedule_block_pairs(1, 1, sta._d3((4, 8, 8)), sta._d3((2, 4, 4)), sta._windows([(1, 1, 1)]),
                                        0, None, 0) == -1


def _call_mixed(lib, q=0x1000000, kt=0x2000000, vt=0x3000000, out=0x4000000, batch=1, heads=1, d=128,
                grid=(11, 22, 37), tile=(6, 8, 8), windows=((1, 3, 3),), scale=0.1):
    return lib.sta_attention_fwd_mixed(q, kt, vt, out, batch, heads, d, sta._d3(grid), sta._d3(tile),
                                       sta._windows(windows), ctypes.c_float(scale), None)


def test_padded_reorder_and_mixed_validation_codes(lib):
    # fake pointers, never dereferenced: validation fails before the device is touched.
    # (11, 22, 37) pads to (12, 24, 40): 8954 raster rows, 11520 tiled rows.
    A, B = 0x1000000, 0x2000000
    pad = lambda src, dst, **kw: lib.sta_tile_reorder_padded(src, dst, kw.get("bh", 1), kw.get("d", 128),  # noqa: E731
                                                             sta._d3(kw.get("grid", (11, 22, 37))),
                                                             sta._d3(kw.get("tile", (6, 8, 8))), None)
    assert pad(None, B) == 1
    assert pad(A + 4, B) == 2
    assert pad(A, A + 8954 * 256 - 16) == 3          # dst starts inside src
    assert pad(A + 11520 * 256 - 16, A) == 3         # src starts inside the (larger) dst
    assert pad(A, B, grid=(0, 22, 37)) == 4
    assert pad(A, B, d=96) == 6
    assert pad(A, B, bh=-1) == 10
    assert _call_mixed(lib, q=None) == 1
    assert _call_mixed(lib, vt=0x3000008) == 2
    assert _call_mixed(lib, out=0x2000000 + 256 * 100) == 3     # out over k_tiled
    assert _call_mixed(lib, tile=(2, 4, 4)) == 4                # 32-token tiles
    assert _call_mixed(lib, tile=(1, 8, 12)) == 4               # not 128-row slabs of whole frames
    assert _call_mixed(lib, windows=((1, 0, 3),)) == 5
    assert _call_mixed(lib, d=48) == 6
    assert _call_mixed(lib, scale=0.0) == 10
    import torch
    if not torch.cuda.is_available():
        # valid arguments and no GPU: a CUDA/architecture error, never a host computation
        assert pad(A, B) in (7, 8)
        assert _call_mixed(lib) in (7, 8)


def _call_host(lib, q=0x1000000, k=0x2000000, v=0x3000000, out=0x4000000, batch=1, heads=1, d=128,
               grid=(12, 24, 40), tile=(6, 8, 8), windows=((1, 3, 3),), scale=0.1, chunk=4):
    return lib.sta_forward_host(q, k, v, out, batch, heads, d, sta._d3(grid), sta._d3(tile), sta._windows(windows),
                                ctypes.c_float(scale), chunk, None)


def test_forward_host_validation_codes(lib):
    codes = {name: code for code, name in sta.STATUS_NAMES.items()}
    assert _call_host(lib, q=0) == codes["STA_ERR_NULL"]
    assert _call_host(lib, d=96) == codes["STA_ERR_HEADDIM"]
    assert _call_host(lib, grid=(4, 8, 8), tile=(2, 4, 4)) == codes["STA_ERR_SHAPE"]   # no 128-row slabs
    assert _call_host(lib, windows=((0, 3, 3),)) == codes["STA_ERR_WINDOW"]
    assert _call_host(lib, chunk=0) == codes["STA_ERR_ARG"]
    assert _call_host(lib, batch=0) == codes["STA_ERR_ARG"]
    assert _call_host(lib, scale=-1.0) == codes["STA_ERR_ARG"]
    assert _call_host(lib, out=0x1000000 + 64) == codes["STA_ERR_ALIAS"]
