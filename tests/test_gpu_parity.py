"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerance (bf16 inputs, fp32 accumulation, bf16 output): max |O_gpu - O_ref|
<= 1e-2 and ||O_gpu - O_ref||_F / ||O_ref||_F <= 5e-3, on every compared row.
Index maps and reorders are compared bit-exactly.  Inputs come from the seeded
generators in ``workloads``; expected values come from ``oracle`` only.
"""
import numpy as np
import pytest
import torch

import oracle.sta_oracle as O
import workloads as W
import sparse_attention_video_tile_b200 as sta

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_FRO = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_video_tile_b200.build import build
    build()
    sta.load_library()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _run_gpu(cfg, q, k, v, fused=None):
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    out = sta.sta_forward(qd, kd, vd, cfg.grid, cfg.tile, cfg.windows, cfg.scale, fused=fused)
    assert sta.sta_check_device_status() == sta.STA_OK
    return out


def _compare(got, want, what):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max abs {err.max():.3e}"
    assert rel <= REL_FRO, f"{what}: rel Frobenius {rel:.3e}"
    return err.max(), rel


def _full_parity(cfg, seed=0, fused=None, pad=False):
    q, k, v = W.make_qkv(cfg, seed)
    out = _run_gpu(cfg, q, k, v, fused).float().cpu().numpy()
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            want = O.sta_attention_head(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                        v[b, h].double().numpy(), cfg.grid, cfg.tile, cfg.windows[h], cfg.scale,
                                        pad=pad)
            _compare(out[b, h], want, f"{cfg.name} b{b} h{h}")


# ------------------------------------------------------------------ reorder


@pytest.mark.parametrize("name", ["tiny", "small", "image2d", "hunyuan", "perhead"])
def test_reorder_unorder_bit_exact(name):
    cfg = W.CONFIGS[name]
    g = torch.Generator(device="cuda").manual_seed(1)
    shape = (cfg.batch, cfg.heads, cfg.L, cfg.d)
    x = torch.randn(shape, device="cuda", generator=g).to(torch.bfloat16)
    y = torch.empty_like(x)
    sta.sta_tile_reorder(x, y, cfg.grid, cfg.tile)
    m = torch.from_numpy(O.tiled_of_raster(cfg.grid, cfg.tile)).cuda()
    want = torch.empty_like(x)
    want[:, :, m, :] = x
    assert torch.equal(y, want)
    z = torch.empty_like(x)
    sta.sta_tile_unorder(y, z, cfg.grid, cfg.tile)
    assert torch.equal(z, x)
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", ["tiny", "small", "image2d", "hunyuan"])
def test_token_major_reorder_bit_exact(name):
    """[B, L, heads, d] raster <-> [B, heads, L, d] tiled, against indexing with the
    oracle's tile map."""
    cfg = W.CONFIGS[name]
    g = torch.Generator(device="cuda").manual_seed(2)
    x = torch.randn((cfg.batch, cfg.L, cfg.heads, cfg.d), device="cuda", generator=g).to(torch.bfloat16)
    y = torch.empty((cfg.batch, cfg.heads, cfg.L, cfg.d), device="cuda", dtype=torch.bfloat16)
    sta.sta_tile_reorder_tokens(x, y, cfg.grid, cfg.tile)
    m = torch.from_numpy(O.tiled_of_raster(cfg.grid, cfg.tile)).cuda()
    want = torch.empty_like(y)
    want[:, :, m, :] = x.transpose(1, 2)
    assert torch.equal(y, want)
    del want
    z = torch.full_like(x, float("nan"))
    sta.sta_tile_unorder_tokens(y, z, cfg.grid, cfg.tile)
    assert torch.equal(z, x)
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_forward_tokens_equals_forward(name):
    """The token-major forward is the head-major forward with both transposes
    folded into the reorders: equal bit for bit."""
    cfg = W.CONFIGS[name]
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, 0))
    want = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale, fused=False)
    tq, tk, tv = (x.transpose(1, 2).contiguous() for x in (q, k, v))
    got = sta.sta_forward_tokens(tq, tk, tv, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    torch.cuda.synchronize()
    assert sta.sta_check_device_status() == sta.STA_OK
    assert got.shape == tq.shape
    assert torch.equal(got.transpose(1, 2), want)


# ------------------------------------------------------------------ attention, full outputs


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_attention_full_parity(name):
    _full_parity(W.CONFIGS[name])


def test_attention_small_three_call_path():
    """The tiled-order path (reorder, attention, unorder) on the small workload."""
    _full_parity(W.CONFIGS["small"], fused=False)


@pytest.mark.parametrize("name", ["small", "image2d"])
def test_fused_raster_path_equals_three_call_path(name):
    """Same schedule and arithmetic: the fused raster kernel must reproduce the
    reorder + tiled attention + unorder path bit for bit on tile-multiple grids."""
    cfg = W.CONFIGS[name]
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, 2))
    a = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale, fused=True)
    b = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale, fused=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


PADDED = [
    # padding with masking: latents that are not tile multiples
    W.custom_config("pad_small", 1, 2, 128, (11, 22, 37), (6, 8, 8), [(1, 3, 3), (3, 3, 3)]),
    W.custom_config("pad_d64", 1, 2, 64, (5, 9, 14), (2, 8, 8), [(1, 1, 1), (3, 3, 3)]),
    W.custom_config("pad_image", 2, 2, 128, (1, 30, 45), (1, 8, 16), [(1, 5, 3), (1, 3, 3)]),
    W.custom_config("pad_perhead", 1, 3, 128, (13, 17, 20), (6, 8, 8), [(1, 3, 3), (3, 5, 5), (5, 6, 10)]),
]


@pytest.mark.parametrize("cfg", PADDED, ids=lambda c: c.name)
def test_attention_padded_latents(cfg):
    _full_parity(cfg, seed=6, pad=True)


def _padded_tiled_reference(x, grid, tile):
    """The oracle's construction of the padded latent's tiled order: zero tokens
    added up to tile multiples, then the tile map of that grid."""
    T, H, Wd = grid
    Tp, Hp, Wp = (-(-a // b) * b for a, b in zip(grid, tile))
    lead = x.shape[:-2]
    d = x.shape[-1]
    full = torch.zeros(lead + (Tp, Hp, Wp, d), dtype=x.dtype, device=x.device)
    full[..., :T, :H, :Wd, :] = x.reshape(lead + (T, H, Wd, d))
    full = full.reshape(lead + (Tp * Hp * Wp, d))
    m = torch.from_numpy(O.tiled_of_raster((Tp, Hp, Wp), tile)).to(x.device)
    out = torch.empty_like(full)
    out[..., m, :] = full
    return out


@pytest.mark.parametrize("cfg", PADDED + [W.CONFIGS["small"]], ids=lambda c: c.name)
def test_padded_reorder_bit_exact(cfg):
    g = torch.Generator(device="cuda").manual_seed(3)
    x = torch.randn((cfg.batch, cfg.heads, cfg.L, cfg.d), device="cuda", generator=g).to(torch.bfloat16)
    y = torch.full((cfg.batch, cfg.heads, sta.padded_rows(cfg.grid, cfg.tile), cfg.d), float("nan"),
                   device="cuda", dtype=torch.bfloat16)
    sta.sta_tile_reorder_padded(x, y, cfg.grid, cfg.tile)
    assert torch.equal(y, _padded_tiled_reference(x, cfg.grid, cfg.tile))
    if cfg.grid[0] % cfg.tile[0] == 0 and cfg.grid[1] % cfg.tile[1] == 0 and cfg.grid[2] % cfg.tile[2] == 0:
        z = torch.empty_like(x)
        sta.sta_tile_reorder(x, z, cfg.grid, cfg.tile)
        assert torch.equal(y, z)
    torch.cuda.synchronize()


@pytest.mark.parametrize("cfg", PADDED, ids=lambda c: c.name)
def test_mixed_path_padded_latents(cfg):
    """Raster q and output, padded tiled k and v: every row against the oracle, and
    bit for bit the one-launch raster path (same schedule and arithmetic)."""
    q, k, v = W.make_qkv(cfg, 6)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    got = sta.sta_forward(qd, kd, vd, cfg.grid, cfg.tile, cfg.windows, cfg.scale, path="mixed")
    ref = sta.sta_forward(qd, kd, vd, cfg.grid, cfg.tile, cfg.windows, cfg.scale, path="fused")
    torch.cuda.synchronize()
    assert sta.sta_check_device_status() == sta.STA_OK
    assert torch.equal(got, ref)
    out = got.float().cpu().numpy()
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            want = O.sta_attention_head(q[b, h].double().numpy(), k[b, h].double().numpy(), v[b, h].double().numpy(),
                                        cfg.grid, cfg.tile, cfg.windows[h], cfg.scale, pad=True)
            _compare(out[b, h], want, f"{cfg.name} mixed b{b} h{h}")


@pytest.mark.parametrize("name", ["small", "image2d", "hunyuan"])
def test_mixed_path_equals_three_call_path(name):
    cfg = W.CONFIGS[name]
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, 2))
    a = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale, path="mixed")
    b = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale, path="three_call")
    torch.cuda.synchronize()
    assert sta.sta_check_device_status() == sta.STA_OK
    assert torch.equal(a, b)


LSE_ABS = 1e-3   # fp32 scores from bf16 inputs, MUFU exponentials, fp32 sums: about 1e-5 expected


@pytest.mark.parametrize("name", ["tiny", "small", "batch2_perhead"])
def test_attention_lse(name):
    """The forward's per-row log-sum-exp against the oracle's, and the output
    unchanged by asking for it."""
    cfg = W.CONFIGS[name] if name in W.CONFIGS else \
        W.custom_config(name, 2, 3, 128, (4, 16, 24), (2, 8, 8), [(1, 1, 1), (3, 3, 3), (1, 2, 3)])
    q, k, v = W.make_qkv(cfg, 4)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    qt, kt, vt = (torch.empty_like(x) for x in (qd, kd, vd))
    for src, dst in ((qd, qt), (kd, kt), (vd, vt)):
        sta.sta_tile_reorder(src, dst, cfg.grid, cfg.tile)
    o1, o2 = torch.empty_like(qt), torch.empty_like(qt)
    lse = torch.full((cfg.batch, cfg.heads, cfg.L), float("nan"), device="cuda", dtype=torch.float32)
    sta.sta_attention_fwd(qt, kt, vt, o1, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    sta.sta_attention_fwd_lse(qt, kt, vt, o2, lse, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    torch.cuda.synchronize()
    assert sta.sta_check_device_status() == sta.STA_OK
    assert torch.equal(o1, o2)
    tiled = O.tiled_of_raster(cfg.grid, cfg.tile)   # raster token n -> tiled row
    got = lse.cpu().numpy().astype(np.float64)
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            want = O.sta_lse_head(q[b, h].double().numpy(), k[b, h].double().numpy(), cfg.grid, cfg.tile,
                                  cfg.windows[h], cfg.scale)
            err = np.abs(got[b, h][tiled] - want)
            assert np.all(np.isfinite(got[b, h])), f"{name} b{b} h{h}: non-finite lse"
            assert err.max() <= LSE_ABS, f"{name} b{b} h{h}: lse max abs {err.max():.3e}"


def test_attention_tiny_other_seeds():
    for seed in (1, 2):
        _full_parity(W.CONFIGS["tiny"], seed)


STRESS = [
    # d = 64 on the mask-free path (Ntile = 128)
    W.custom_config("d64_fast", 1, 2, 64, (4, 16, 16), (2, 8, 8), [(1, 3, 3), (3, 3, 3)]),
    # even windows: the window reaches one tile further below the query tile
    W.custom_config("even", 1, 3, 128, (6, 16, 32), (2, 8, 8), [(2, 2, 2), (3, 1, 4), (1, 2, 3)]),
    # window larger than the grid (dense) and a single tile
    W.custom_config("wide", 1, 1, 128, (6, 16, 16), (2, 8, 8), [(9, 9, 9)]),
    W.custom_config("single_tile", 1, 2, 128, (6, 8, 8), (6, 8, 8), [(1, 1, 1), (3, 3, 3)]),
    # batch > 1 with per-head windows
    W.custom_config("batch2", 2, 3, 128, (4, 16, 24), (2, 8, 8), [(1, 1, 1), (3, 3, 3), (1, 2, 3)]),
    # Ntile = 256 (two blocks per tile)
    W.custom_config("ntile256", 1, 2, 128, (4, 16, 32), (1, 16, 16), [(3, 1, 1), (1, 1, 2)]),
    # masked path: small tiles, L not a multiple of 128 (ragged last block)
    W.custom_config("ragged25", 1, 2, 64, (3, 10, 10), (1, 5, 5), [(1, 1, 1), (3, 1, 2)]),
    W.custom_config("ragged32", 1, 2, 128, (2, 12, 12), (2, 4, 4), [(1, 3, 3), (1, 2, 1)]),
    W.custom_config("ntile64", 2, 2, 128, (4, 16, 16), (1, 8, 8), [(3, 3, 3), (1, 1, 2)]),
]


@pytest.mark.parametrize("cfg", STRESS, ids=lambda c: c.name)
def test_attention_stress_shapes(cfg):
    _full_parity(cfg, seed=3)


# Many work items per CTA, every row against the oracle.  18 heads of the small
# latent give 18 x 90 = 1620 query blocks on a grid of one CTA per SM (about 11
# items per CTA on 148 SMs).  The mixed windows make items of 3 to 27 key blocks,
# so item boundaries come often: each one hands O from the epilogue of one item
# to the first, overwriting P V of the next, and every such hand-over is checked.
MANY_ITEMS = W.custom_config("many_items", 1, 18, 128, (12, 24, 40), (6, 8, 8),
                             [(1, 1, 1), (3, 3, 3), (1, 3, 3), (2, 3, 5), (1, 2, 1), (3, 1, 2)] * 3)


@pytest.mark.parametrize("fused", [False, True], ids=["three_call", "fused"])
def test_attention_many_items_per_cta_full_oracle(fused):
    _full_parity(MANY_ITEMS, seed=21, fused=fused)


def test_attention_hunyuan_bitwise_repeatable():
    """Five full forwards of the HunyuanVideo-shaped workload give the same bits:
    a race between the pipeline's agents would show up as run-to-run differences."""
    cfg = W.CONFIGS["hunyuan"]
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, 3))
    first = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale, fused=False)
    for _ in range(4):
        again = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale, fused=False)
        torch.cuda.synchronize()
        assert torch.equal(again, first)
        del again
    assert sta.sta_check_device_status() == sta.STA_OK


# ------------------------------------------------------------------ attention, sampled rows at full size


def _sampled_parity(cfg, heads, seed=0):
    q, k, v = W.make_qkv(cfg, seed)
    out = _run_gpu(cfg, q, k, v)
    rows = W.sample_rows(cfg, seed)
    rows_t = torch.tensor(rows, device="cuda")
    for b, h in heads:
        got = out[b, h].index_select(0, rows_t).float().cpu().numpy()
        want = O.sta_attention_head(q[b, h].double().numpy(), k[b, h].double().numpy(), v[b, h].double().numpy(),
                                    cfg.grid, cfg.tile, cfg.windows[h], cfg.scale, rows=rows)
        _compare(got, want, f"{cfg.name} b{b} h{h}")
    # every output row is finite and bounded by the value range
    assert torch.isfinite(out.float()).all()


def test_attention_hunyuan_sampled():
    _sampled_parity(W.CONFIGS["hunyuan"], [(0, 0), (0, 11), (0, 23)])


def test_attention_image2d_sampled():
    _sampled_parity(W.CONFIGS["image2d"], [(0, 0), (1, 17)])


def test_attention_hunyuan_padded_sampled():
    """The review reply's example: a (29, 45, 76) latent padded to (30, 48, 80)."""
    cfg = W.custom_config("hunyuan_pad", 1, 2, 128, (29, 45, 76), (6, 8, 8), [(3, 3, 3)])
    q, k, v = W.make_qkv(cfg, 0)
    out = _run_gpu(cfg, q, k, v)
    rows = W.sample_rows(cfg, 0)
    rows_t = torch.tensor(rows, device="cuda")
    for h in range(cfg.heads):
        got = out[0, h].index_select(0, rows_t).float().cpu().numpy()
        want = O.sta_attention_head(q[0, h].double().numpy(), k[0, h].double().numpy(), v[0, h].double().numpy(),
                                    cfg.grid, cfg.tile, cfg.windows[h], cfg.scale, rows=rows, pad=True)
        _compare(got, want, f"hunyuan_pad h{h}")
    assert torch.isfinite(out.float()).all()


def test_attention_hunyuan_three_call_path_sampled():
    cfg = W.CONFIGS["hunyuan"]
    q, k, v = W.make_qkv(cfg, 1)
    out = _run_gpu(cfg, q, k, v, fused=False)
    rows = W.sample_rows(cfg, 1)
    rows_t = torch.tensor(rows, device="cuda")
    got = out[0, 5].index_select(0, rows_t).float().cpu().numpy()
    want = O.sta_attention_head(q[0, 5].double().numpy(), k[0, 5].double().numpy(), v[0, 5].double().numpy(),
                                cfg.grid, cfg.tile, cfg.windows[5], cfg.scale, rows=rows)
    _compare(got, want, "hunyuan three-call h5")


def test_attention_perhead_sampled():
    cfg = W.CONFIGS["perhead"]
    seen, heads = set(), []
    for h, w in enumerate(cfg.windows):
        if w not in seen:
            seen.add(w)
            heads.append((0, h))
    _sampled_parity(cfg, heads)


def test_attention_score_jumps_exercise_rescale_paths():
    """Planted keys whose scores jump far above the running max in a later block.

    The kernel moves a row's running max only when a block's max exceeds it by more
    than 2^8, and then rescales O and the row sum together.  Random N(0, 1) inputs
    never get there.  Two query rows of an interior tile get one planted key each,
    scoring about 110 (log2 units) above the rest, inside their own tile (never the
    first block of the window): one in the first 64 keys of a 128-key block and one
    in the last 64.
    """
    cfg = W.custom_config("jumps", 1, 1, 128, (12, 24, 40), (6, 8, 8), [(1, 3, 3)])
    q, k, v = W.make_qkv(cfg, 11)
    # Rows dominated by one planted key output that key's value row; scaling v keeps
    # those outputs in the magnitude range the absolute tolerance is stated for (bf16
    # rounding of P and of the output is relative).  A wrong rescale factor would be
    # off by 2^8 or more.
    v = (v.float() * 0.25).to(torch.bfloat16)
    T, H, Wd = cfg.grid
    m = O.tiled_of_raster(cfg.grid, cfg.tile)
    inv = np.empty_like(m)
    inv[m] = np.arange(m.size)
    tile_id = (1 * 3 + 1) * 5 + 2          # tile (1, 1, 2): interior in H and W
    base = tile_id * cfg.ntile
    for q_local, k_local in ((200, 10), (300, 100)):
        nq, nk = int(inv[base + q_local]), int(inv[base + k_local])
        qa = q[0, 0, nq].double()
        lam = 110.0 / (1.4426950408889634 * cfg.scale)   # scaled score of ~110 in log2 units
        k[0, 0, nk] = (qa * (lam / float(qa @ qa))).to(torch.bfloat16)
    out = _run_gpu(cfg, q, k, v).float().cpu().numpy()
    want = O.sta_attention_head(q[0, 0].double().numpy(), k[0, 0].double().numpy(), v[0, 0].double().numpy(),
                                cfg.grid, cfg.tile, cfg.windows[0], cfg.scale)
    _compare(out[0, 0], want, "planted score jumps")


@pytest.mark.parametrize("poly8", ["1"])
def test_attention_fma_pipe_exp2_variants(poly8):
    """Some exponentials on the FMA pipe (cubic minimax 2^f on packed pairs): same tolerance."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, STA_EXP_POLY8=poly8)
    here = os.path.dirname(os.path.abspath(__file__))
    r = subprocess.run([sys.executable, os.path.join(here, "gpu_poly_check.py"), "small"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr


# ------------------------------------------------------------------ behaviour


def test_deterministic_and_inputs_untouched():
    cfg = W.CONFIGS["small"]
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, 4))
    q0, k0, v0 = q.clone(), k.clone(), v.clone()
    a = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    b = sta.sta_forward(q, k, v, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(q, q0) and torch.equal(k, k0) and torch.equal(v, v0)


def test_misaligned_pointer_rejected():
    cfg = W.CONFIGS["tiny"]
    buf = torch.zeros(cfg.heads * cfg.L * cfg.d + 1, dtype=torch.bfloat16, device="cuda")
    x = buf[1:].view(1, cfg.heads, cfg.L, cfg.d)
    y = torch.empty_like(x)
    with pytest.raises(sta.StaError) as e:
        sta.sta_tile_reorder(x, y, cfg.grid, cfg.tile)
    assert e.value.status == 2


def test_bounded_wait_gives_up_and_context_survives():
    # a barrier that nothing completes: the kernel must give up and say so
    assert sta.sta_selftest_bounded_wait(20_000_000) == sta.STA_ERR_TIMEOUT
    # the flag is cleared and the library still computes correctly
    assert sta.sta_check_device_status() == sta.STA_OK
    _full_parity(W.CONFIGS["tiny"])


def test_forward_from_host_equals_device_forward():
    """The copy-overlapped host entry gives, head by head, the device forward's bits."""
    cfg = W.custom_config("host_b2", 2, 5, 128, (12, 24, 40), (6, 8, 8),
                          [(1, 3, 3), (3, 3, 3), (1, 1, 1), (3, 5, 5), (1, 3, 3)])
    q, k, v = W.make_qkv(cfg, 12)
    want = sta.sta_forward(q.cuda(), k.cuda(), v.cuda(), cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    out_h = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    sta.sta_forward_from_host(qh, kh, vh, out_h, cfg.grid, cfg.tile, cfg.windows, cfg.scale, heads_per_chunk=2)
    assert sta.sta_check_device_status() == sta.STA_OK
    assert torch.equal(out_h, want.cpu())


def test_forward_host_pageable_padded_latent():
    """The C-ABI host entry on pageable host memory (copies that do not overlap) and a
    latent that is not a tile multiple (padded inside, real tokens only in and out),
    three heads in chunks of two: the device forward's bits, head by head."""
    cfg = W.custom_config("host_padded", 1, 3, 128, (11, 22, 37), (6, 8, 8), [(1, 3, 3), (3, 3, 3), (1, 1, 1)])
    q, k, v = W.make_qkv(cfg, 21)
    want = sta.sta_forward(q.cuda(), k.cuda(), v.cuda(), cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    out_h = torch.empty(q.shape, dtype=q.dtype)
    sta.sta_forward_host(q, k, v, out_h, cfg.grid, cfg.tile, cfg.windows, cfg.scale, heads_per_chunk=2)
    assert sta.sta_check_device_status() == sta.STA_OK
    assert torch.equal(out_h, want.cpu())


def test_schedule_cache_eviction_with_launches_in_flight():
    """More configurations than the library's schedule cache holds, launched back to back
    with one synchronize at the end: evicting a schedule must not free arrays that a
    queued kernel still reads.  Every output is checked against the oracle."""
    grids = [(4, 8, 8), (6, 8, 8), (4, 12, 8)]
    windows = [(a, b, c) for a in (1, 3) for b in (1, 3) for c in (1, 3)]
    runs = []
    for gi, grid in enumerate(grids):
        for wi, win in enumerate(windows):
            cfg = W.custom_config(f"evict_{gi}_{wi}", 1, 1, 64, grid, (2, 4, 4), [win])
            q, k, v = W.make_qkv(cfg, 100 + 8 * gi + wi)
            out = sta.sta_forward(q.cuda(), k.cuda(), v.cuda(), cfg.grid, cfg.tile, cfg.windows, cfg.scale)
            runs.append((cfg, q, k, v, out))
    assert len(runs) > 16
    torch.cuda.synchronize()
    assert sta.sta_check_device_status() == sta.STA_OK
    for cfg, q, k, v, out in runs:
        want = O.sta_attention_head(q[0, 0].double().numpy(), k[0, 0].double().numpy(),
                                    v[0, 0].double().numpy(), cfg.grid, cfg.tile, cfg.windows[0], cfg.scale)
        _compare(out[0, 0].float().cpu().numpy(), want, cfg.name)
