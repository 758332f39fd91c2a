"""GPU parity of the backward pass (through the C ABI) against the fp64 oracle.

The oracle's backward is the chain rule of masked softmax attention, pinned by
autograd, finite differences and closed forms (oracle_pins.py).  The CUDA path
takes bf16 operands, accumulates in fp32, rounds P and dS to bf16 for the
products that take them and rounds dq, dk, dv to bf16.  Each of those roundings
is a relative error of at most 2^-9 per element, so the relative Frobenius error
of a gradient is a small multiple of 2^-9 (about 2.4e-3 measured on B200);
the bounds below allow 5e-3, and for the largest element error 1 % of the
gradient's largest magnitude.
"""
import numpy as np
import pytest
import torch

import oracle.sta_oracle as O
import workloads as W
import sparse_attention_video_tile_b200 as sta

pytestmark = pytest.mark.gpu

REL_FRO = 5e-3
MAX_REL_TO_PEAK = 1e-2


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


def _gpu_backward(cfg, seed):
    """Forward (with log-sum-exp) and backward on tiled tensors; gradients returned in
    raster order, with the raster inputs and output gradient."""
    q, k, v = W.make_qkv(cfg, seed)
    do = W.make_qkv(cfg, seed + 100)[0]
    dev = [x.cuda() for x in (q, k, v, do)]
    qt, kt, vt, dot = (torch.empty_like(x) for x in dev)
    for src, dst in zip(dev, (qt, kt, vt, dot)):
        sta.sta_tile_reorder(src, dst, cfg.grid, cfg.tile)
    ot = torch.empty_like(qt)
    lse = torch.empty(cfg.batch, cfg.heads, cfg.L, device="cuda", dtype=torch.float32)
    sta.sta_attention_fwd_lse(qt, kt, vt, ot, lse, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    grads = [torch.full_like(qt, float("nan")) for _ in range(3)]
    sta.sta_attention_bwd(qt, kt, vt, ot, dot, lse, *grads, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    torch.cuda.synchronize()
    assert sta.sta_check_device_status() == sta.STA_OK
    raster = []
    for g in grads:
        r = torch.empty_like(g)
        sta.sta_tile_unorder(g, r, cfg.grid, cfg.tile)
        raster.append(r)
    torch.cuda.synchronize()
    return (q, k, v, do), [r.float().cpu().numpy().astype(np.float64) for r in raster]


def _compare(got, want, what):
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    peak = np.abs(want).max()
    worst = np.abs(got - want).max()
    assert rel <= REL_FRO, f"{what}: rel Frobenius {rel:.3e}"
    assert worst <= MAX_REL_TO_PEAK * peak, f"{what}: max abs {worst:.3e} vs peak {peak:.3e}"


CASES = [
    W.CONFIGS["small"],
    W.custom_config("bwd_b2_d64", 2, 3, 64, (4, 16, 24), (2, 8, 8), [(1, 1, 1), (3, 3, 3), (1, 2, 3)]),
    W.custom_config("bwd_image", 1, 2, 128, (1, 32, 48), (1, 8, 16), [(1, 3, 3), (1, 4, 2)]),
    W.custom_config("bwd_dense", 1, 1, 128, (6, 16, 16), (6, 8, 8), [(1, 9, 9)]),   # window covers the grid
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_backward_full_parity(cfg):
    (q, k, v, do), got = _gpu_backward(cfg, seed=5)
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            want = O.sta_attention_backward_head(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                                 v[b, h].double().numpy(), do[b, h].double().numpy(),
                                                 cfg.grid, cfg.tile, cfg.windows[h], cfg.scale)
            for name, g, w in zip(("dq", "dk", "dv"), (x[b, h] for x in got), want):
                _compare(g, w, f"{cfg.name} b{b} h{h} {name}")


def _key_tile_rows(cfg, a):
    """Raster rows of the tokens of tile a = (at, ah, aw)."""
    T, H, Wd = cfg.grid
    tt, th, tw = cfg.tile
    t, h, w = np.meshgrid(np.arange(a[0] * tt, (a[0] + 1) * tt), np.arange(a[1] * th, (a[1] + 1) * th),
                          np.arange(a[2] * tw, (a[2] + 1) * tw), indexing="ij")
    return np.sort(((t * H + h) * Wd + w).ravel())


def _dk_dv_of_key_tile(cfg, q64, k64, v64, do64, window, a):
    """Exact dk, dv of the keys of tile a from the oracle's chain rule.  Only the
    query rows whose window contains tile a have P != 0 on its keys, so they alone
    contribute; each takes its softmax over its own window, for which the keys of
    the union of those windows suffice (the mask removes the rest)."""
    coords = O.raster_coords(cfg.grid)
    krows = _key_tile_rows(cfg, a)
    queries = np.nonzero(O.sta_mask(coords, coords[krows[:1]], cfg.grid, cfg.tile, window)[:, 0])[0]
    union = np.zeros(cfg.L, dtype=bool)
    for r0 in range(0, queries.size, 2048):
        union |= O.sta_mask(coords[queries[r0:r0 + 2048]], coords, cfg.grid, cfg.tile, window).any(axis=0)
    keys = np.nonzero(union)[0]
    pos = np.searchsorted(keys, krows)
    assert np.array_equal(keys[pos], krows)
    dk = np.zeros((krows.size, k64.shape[1]))
    dv = np.zeros((krows.size, v64.shape[1]))
    for r0 in range(0, queries.size, 512):
        sel = queries[r0:r0 + 512]
        mask = O.sta_mask(coords[sel], coords[keys], cfg.grid, cfg.tile, window)
        _, gk, gv = O.masked_softmax_attention_backward(q64[sel], k64[keys], v64[keys], mask, cfg.scale, do64[sel])
        dk += gk[pos]
        dv += gv[pos]
    return krows, dk, dv


def test_backward_hunyuan_full_size_dq_rows_and_dk_dv_tiles():
    """At the full 30x48x80 size: dq of sampled rows (a row's dq needs only its own
    window), dk and dv element by element on one whole key tile per head (an
    interior tile and a corner tile), and the closed forms sum_k dv = sum_q dO and
    sum_k dk = 0 over all keys."""
    cfg = W.CONFIGS["hunyuan"]
    cases = ((0, (2, 3, 5)), (13, (0, 0, 0)))
    (q, k, v, do), got = _gpu_backward(cfg, seed=7)
    rng = np.random.default_rng(3)
    coords = O.raster_coords(cfg.grid)
    for h, a in cases:
        rows = np.sort(rng.choice(cfg.L, 48, replace=False))
        q64, k64, v64, do64 = (x[0, h].double().numpy() for x in (q, k, v, do))
        mask = O.sta_mask(coords[rows], coords, cfg.grid, cfg.tile, cfg.windows[h])
        want_dq, _, _ = O.masked_softmax_attention_backward(q64[rows], k64, v64, mask, cfg.scale, do64[rows])
        _compare(got[0][0, h][rows], want_dq, f"hunyuan h{h} dq rows")
        krows, want_dk, want_dv = _dk_dv_of_key_tile(cfg, q64, k64, v64, do64, cfg.windows[h], a)
        _compare(got[1][0, h][krows], want_dk, f"hunyuan h{h} dk of tile {a}")
        _compare(got[2][0, h][krows], want_dv, f"hunyuan h{h} dv of tile {a}")
        dv_sum, do_sum = got[2][0, h].sum(axis=0), do64.sum(axis=0)
        assert np.abs(dv_sum - do_sum).max() <= 1e-2 * np.abs(do_sum).max() + 0.5
        assert np.abs(got[1][0, h].sum(axis=0)).max() <= 1e-2 * np.abs(got[1][0, h]).sum(axis=0).max() + 0.5


# ------------------------------------------------------------------ autograd wrapper

AUTOGRAD_CFG = W.custom_config("autograd", 1, 2, 64, (4, 16, 16), (2, 8, 8), [(1, 1, 1), (2, 2, 1)])


def test_autograd_matches_oracle_and_explicit_calls():
    """sta_attention's forward and gradients: the same values as the explicit C-ABI
    calls (bit for bit) and as the oracle (within the tolerances above)."""
    from sparse_attention_video_tile_b200.autograd import sta_attention
    cfg = AUTOGRAD_CFG
    (q, k, v, do), want_explicit = _gpu_backward(cfg, 3)
    leaves = [x.cuda().requires_grad_(True) for x in (q, k, v)]
    out = sta_attention(*leaves, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    out.backward(do.cuda())
    torch.cuda.synchronize()
    assert sta.sta_check_device_status() == sta.STA_OK
    want_out = sta.sta_forward(q.cuda(), k.cuda(), v.cuda(), cfg.grid, cfg.tile, cfg.windows, cfg.scale,
                               fused=False)
    assert torch.equal(out.detach(), want_out)
    got = [x.grad.float().cpu().numpy().astype(np.float64) for x in leaves]
    for name, g, e in zip(("dq", "dk", "dv"), got, want_explicit):
        assert np.array_equal(g, e), f"{name}: autograd differs from the explicit calls"
    for h in range(cfg.heads):
        want = O.sta_attention_backward_head(*(x[0, h].double().numpy() for x in (q, k, v, do)),
                                             cfg.grid, cfg.tile, cfg.windows[h], cfg.scale)
        for name, g, w in zip(("dq", "dk", "dv"), got, want):
            _compare(g[0, h], w, f"autograd head {h} {name}")


def test_autograd_token_major_equals_head_major():
    from sparse_attention_video_tile_b200.autograd import sta_attention
    cfg = AUTOGRAD_CFG
    q, k, v = (x.cuda() for x in W.make_qkv(cfg, 4))
    do = W.make_qkv(cfg, 5)[0].cuda()
    a = [x.clone().requires_grad_(True) for x in (q, k, v)]
    b = [x.transpose(1, 2).contiguous().requires_grad_(True) for x in (q, k, v)]
    out_a = sta_attention(*a, cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    out_b = sta_attention(*b, cfg.grid, cfg.tile, cfg.windows, cfg.scale, token_major=True)
    out_a.backward(do)
    out_b.backward(do.transpose(1, 2))     # a non-contiguous gradient: the wrapper makes it contiguous
    torch.cuda.synchronize()
    assert sta.sta_check_device_status() == sta.STA_OK
    assert torch.equal(out_b.detach().transpose(1, 2), out_a.detach())
    for x, y in zip(a, b):
        assert torch.equal(y.grad.transpose(1, 2), x.grad)
