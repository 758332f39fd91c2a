"""Pins for the CPU oracle: checks against facts that do not come from the oracle.

Each ``pin_*`` takes the oracle module so that the mutation tests can run the
same checks against an oracle with a planted mistake and see them fail.

Sources of the facts pinned here:
  * hand-worked fixtures under tests/golden/ (each cites its passage);
  * brute-force enumeration of window membership written as plain loops with a
    different formulation of the window rule (the feasible window whose centre
    tile is closest to the query tile);
  * closed forms: pair counts L * Ntile * prod(min(w, n)), the uniform-softmax
    case (q = 0 gives the mean of the attended value rows);
  * library routines for the special cases that reduce to plain attention
    (window covering the grid = dense attention; window (1,1,1) = attention
    inside each tile), computed with torch's scaled_dot_product_attention in
    fp64;
  * invariants: permutation of tokens, rows of P summing to one, outputs inside
    the hull of the attended value rows;
  * for the log-sum-exp and the backward: torch.logsumexp and torch autograd of
    masked scaled_dot_product_attention over the brute-force window, central
    finite differences through the forward, and the closed-form gradient sums.
"""
from __future__ import annotations

import os
import itertools

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


def _rand_qkv(L, d, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(L, d, generator=g, dtype=torch.float64) for _ in range(3))
    return q.numpy(), k.numpy(), v.numpy()


# ----------------------------------------------------------------------------- index map


def pin_index_map_golden(o):
    rows = _read_golden("index_map_grid2x2x4_tile1x2x2.txt")
    kv = {r.split()[0]: [int(x) for x in r.split()[1:]] for r in rows}
    got = o.tiled_of_raster(kv["grid"], kv["tile"])
    assert got.tolist() == kv["map"], (got.tolist(), kv["map"])


def pin_index_map_properties(o):
    shapes = [((4, 8, 8), (2, 4, 4)), ((12, 24, 40), (6, 8, 8)), ((1, 16, 16), (1, 8, 16)),
              ((3, 5, 7), (1, 5, 7)), ((6, 4, 10), (3, 2, 5))]
    for grid, tile in shapes:
        m = o.tiled_of_raster(grid, tile)
        L = int(np.prod(grid))
        ntile = int(np.prod(tile))
        assert sorted(m.tolist()) == list(range(L))
        # tokens of one tile occupy one aligned run of Ntile rows, in raster order
        T, H, W = grid
        tt, th, tw = tile
        for at, ah, aw in itertools.product(range(T // tt), range(H // th), range(W // tw)):
            toks = [(t * H + h) * W + w
                    for t in range(at * tt, at * tt + tt)
                    for h in range(ah * th, ah * th + th)
                    for w in range(aw * tw, aw * tw + tw)]
            run = m[toks]
            assert run[0] % ntile == 0
            assert run.tolist() == list(range(run[0], run[0] + ntile))
        # tiles in raster order over the tile grid
        first = [m[(at * tt * H + ah * th) * W + aw * tw]
                 for at, ah, aw in itertools.product(range(T // tt), range(H // th), range(W // tw))]
        assert first == [i * ntile for i in range(len(first))]


def pin_reorder_roundtrip(o):
    grid, tile = (4, 8, 8), (2, 4, 4)
    x = np.arange(2 * 256 * 3, dtype=np.float64).reshape(2, 256, 3)
    y = o.reorder(x, grid, tile)
    m = o.tiled_of_raster(grid, tile)
    for n in range(256):
        assert np.array_equal(y[:, m[n]], x[:, n])
    assert np.array_equal(o.unorder(y, grid, tile), x)


# ----------------------------------------------------------------------------- window rule


def pin_window_golden(o):
    for line in _read_golden("window_clamp_1d.txt"):
        lhs, rhs = line.split(":")
        n, w, a = (int(x) for x in lhs.split())
        want = [int(x) for x in rhs.split()]
        coords = o.raster_coords((1, 1, n))
        mask = o.sta_mask(coords, coords, (1, 1, n), (1, 1, 1), (1, 1, w))
        got = np.nonzero(mask[a])[0].tolist()
        assert got == want, (n, w, a, got, want)


def _brute_window(a, w, n):
    """Key tiles of query tile a: among all feasible windows of min(w, n)
    consecutive tiles pick the one whose centre slot is closest to a."""
    we = w if w < n else n
    best = None
    for s in range(0, n - we + 1):
        dist = abs(s + we // 2 - a)
        if best is None or dist < best[0]:
            best = (dist, s)
    s = best[1]
    return set(range(s, s + we))


def _brute_mask(grid, tile, window, pad=False):
    T, H, W = grid
    tt, th, tw = tile
    toks = []
    for t in range(T):
        for h in range(H):
            for w in range(W):
                toks.append((t, h, w))
    n = ((T + tt - 1) // tt, (H + th - 1) // th, (W + tw - 1) // tw) if pad else (T // tt, H // th, W // tw)
    L = len(toks)
    mask = np.zeros((L, L), dtype=bool)
    for i, (t, h, w) in enumerate(toks):
        a = (t // tt, h // th, w // tw)
        wins = [_brute_window(a[x], window[x], n[x]) for x in range(3)]
        for j, (t2, h2, w2) in enumerate(toks):
            if (t2 // tt) in wins[0] and (h2 // th) in wins[1] and (w2 // tw) in wins[2]:
                mask[i, j] = True
    return mask


BRUTE_CASES = [
    ((4, 8, 8), (2, 4, 4), (1, 1, 1)),
    ((4, 8, 8), (2, 4, 4), (3, 3, 3)),
    ((4, 8, 8), (1, 2, 2), (3, 3, 3)),
    ((4, 8, 8), (1, 2, 2), (2, 4, 2)),
    ((3, 6, 10), (1, 2, 2), (3, 2, 3)),
    ((2, 6, 10), (1, 1, 2), (1, 5, 4)),
    ((1, 8, 12), (1, 2, 2), (1, 3, 9)),
    ((5, 4, 6), (1, 2, 3), (2, 1, 1)),
]


def pin_mask_brute_force(o):
    for grid, tile, window in BRUTE_CASES:
        coords = o.raster_coords(grid)
        got = o.sta_mask(coords, coords, grid, tile, window)
        want = _brute_mask(grid, tile, window)
        assert np.array_equal(got, want), (grid, tile, window)


def _closed_form_pairs(grid, tile, window):
    L = int(np.prod(grid))
    ntile = int(np.prod(tile))
    n = [g // t for g, t in zip(grid, tile)]
    return L * ntile * int(np.prod([min(w, x) for w, x in zip(window, n)]))


def pin_pair_counts(o):
    for grid, tile, window in BRUTE_CASES:
        coords = o.raster_coords(grid)
        mask = o.sta_mask(coords, coords, grid, tile, window)
        cf = _closed_form_pairs(grid, tile, window)
        assert int(mask.sum()) == cf
        assert o.attended_pairs_head(grid, tile, window) == cf
        # every row sees exactly Ntile * prod(w') keys, its own tile included
        assert np.all(mask.sum(axis=1) == cf // int(np.prod(grid)))
        assert np.all(np.diag(mask))
    from workloads import CONFIGS
    golden = dict(line.split() for line in _read_golden("attended_pairs.txt"))
    for name, want in golden.items():
        c = CONFIGS[name]
        assert o.attended_pairs(c.batch, c.grid, c.tile, c.windows) == int(want), name


# ----------------------------------------------------------------------------- attention values


def _sdpa(q, k, v, scale):
    t = [torch.from_numpy(np.ascontiguousarray(x))[None, None] for x in (q, k, v)]
    return torch.nn.functional.scaled_dot_product_attention(*t, scale=scale)[0, 0].numpy()


def pin_dense_equals_library(o):
    for grid, tile, window, d in [((4, 8, 8), (2, 4, 4), (3, 3, 3), 16),
                                  ((2, 6, 10), (1, 2, 2), (9, 9, 9), 8),
                                  ((3, 4, 4), (1, 2, 2), (3, 2, 2), 12)]:
        L = int(np.prod(grid))
        q, k, v = _rand_qkv(L, d, seed=L + d)
        scale = 0.37
        got = o.sta_attention_head(q, k, v, grid, tile, window, scale)
        want = _sdpa(q, k, v, scale)
        assert np.max(np.abs(got - want)) < 1e-12


def pin_window_111_is_per_tile_attention(o):
    grid, tile, d = (4, 8, 8), (2, 4, 4), 16
    L = 256
    q, k, v = _rand_qkv(L, d, seed=5)
    got = o.sta_attention_head(q, k, v, grid, tile, (1, 1, 1), 0.25)
    T, H, W = grid
    tt, th, tw = tile
    for at, ah, aw in itertools.product(range(T // tt), range(H // th), range(W // tw)):
        toks = [(t * H + h) * W + w
                for t in range(at * tt, at * tt + tt)
                for h in range(ah * th, ah * th + th)
                for w in range(aw * tw, aw * tw + tw)]
        want = _sdpa(q[toks], k[toks], v[toks], 0.25)
        assert np.max(np.abs(got[toks] - want)) < 1e-12


def pin_uniform_softmax_mean(o):
    """q = 0 makes every allowed score equal: the output is the plain mean of
    the value rows in the window (closed form)."""
    grid, tile, window, d = (3, 6, 10), (1, 2, 2), (3, 2, 3), 4
    L = int(np.prod(grid))
    _, k, v = _rand_qkv(L, d, seed=11)
    q = np.zeros((L, d))
    got = o.sta_attention_head(q, k, v, grid, tile, window, 1.0)
    mask = _brute_mask(grid, tile, window)
    for i in range(L):
        want = v[mask[i]].mean(axis=0)
        assert np.max(np.abs(got[i] - want)) < 1e-12


def pin_permutation_invariance(o):
    grid, tile, window, d = (4, 8, 8), (1, 2, 2), (3, 3, 2), 8
    L = 256
    q, k, v = _rand_qkv(L, d, seed=3)
    coords = o.raster_coords(grid)
    base = o.masked_softmax_attention(q, k, v, o.sta_mask(coords, coords, grid, tile, window), 0.5)
    # a random permutation applied to tokens and coordinates alike
    perm = np.random.default_rng(7).permutation(L)
    cp = coords[perm]
    out = o.masked_softmax_attention(q[perm], k[perm], v[perm], o.sta_mask(cp, cp, grid, tile, window), 0.5)
    assert np.max(np.abs(out - base[perm])) < 1e-12
    # the tiled order in particular
    m = o.tiled_of_raster(grid, tile)
    inv = np.empty(L, dtype=np.int64)
    inv[m] = np.arange(L)
    ct = coords[inv]
    out_t = o.masked_softmax_attention(o.reorder(q, grid, tile), o.reorder(k, grid, tile),
                                       o.reorder(v, grid, tile), o.sta_mask(ct, ct, grid, tile, window), 0.5)
    assert np.max(np.abs(o.unorder(out_t, grid, tile) - base)) < 1e-12


def pin_rows_normalised_and_hull(o):
    grid, tile, window, d = (3, 6, 10), (1, 2, 2), (2, 3, 3), 8
    L = int(np.prod(grid))
    q, k, v = _rand_qkv(L, d, seed=9)
    coords = o.raster_coords(grid)
    mask = o.sta_mask(coords, coords, grid, tile, window)
    out, p = o.masked_softmax_attention(q, k, v, mask, 0.7, return_p=True)
    assert np.max(np.abs(p.sum(axis=1) - 1.0)) < 1e-12
    assert np.all(p[~mask] == 0.0)
    assert np.all(p[mask] > 0.0)
    for i in range(L):
        vv = v[mask[i]]
        assert np.all(out[i] <= vv.max(axis=0) + 1e-12)
        assert np.all(out[i] >= vv.min(axis=0) - 1e-12)


def pin_sampled_rows_match_full(o):
    grid, tile, window, d = (4, 8, 8), (2, 4, 4), (1, 2, 1), 8
    q, k, v = _rand_qkv(256, d, seed=21)
    full = o.sta_attention_head(q, k, v, grid, tile, window, 0.3)
    rows = [255, 0, 17, 128, 64]
    part = o.sta_attention_head(q, k, v, grid, tile, window, 0.3, rows=rows, row_block=2)
    assert np.max(np.abs(part - full[rows])) < 1e-13


# ----------------------------------------------------------------------------- padding


def pin_padding_golden(o):
    for line in _read_golden("window_padded_1d.txt"):
        lhs, rhs = line.split(":")
        W, t, w, a = (int(x) for x in lhs.split())
        want = [int(x) for x in rhs.split()]
        coords = o.raster_coords((1, 1, W))
        mask = o.sta_mask(coords, coords, (1, 1, W), (1, 1, t), (1, 1, w), pad=True)
        got = np.nonzero(mask[a])[0].tolist()
        assert got == want, (W, t, w, a, got, want)


PAD_CASES = [
    ((5, 7, 9), (2, 4, 4), (1, 1, 1)),
    ((5, 7, 9), (2, 4, 4), (3, 3, 3)),
    ((3, 10, 11), (2, 4, 4), (1, 3, 2)),
    ((4, 9, 6), (3, 2, 4), (2, 3, 1)),
]


def pin_padding_brute_force(o):
    for grid, tile, window in PAD_CASES:
        coords = o.raster_coords(grid)
        got = o.sta_mask(coords, coords, grid, tile, window, pad=True)
        want = _brute_mask(grid, tile, window, pad=True)
        assert np.array_equal(got, want), (grid, tile, window)
        assert int(got.sum()) == o.attended_pairs_head(grid, tile, window, pad=True)


def pin_padding_equals_explicit_padded_grid(o):
    """Pad the latent explicitly (zero tokens) to a tile multiple, attend on the
    padded grid with the unpadded rule while masking pad keys, keep real rows."""
    for (grid, tile, window), d in zip(PAD_CASES, (8, 16, 8, 12)):
        L = int(np.prod(grid))
        q, k, v = _rand_qkv(L, d, seed=L)
        gp = tuple(-(-g // t) * t for g, t in zip(grid, tile))
        Lp = int(np.prod(gp))
        cp = o.raster_coords(gp)
        real = np.all(cp < np.array(grid), axis=1)
        qp, kp, vp = (np.zeros((Lp, d)) for _ in range(3))
        idx = np.nonzero(real)[0]  # padded raster positions of the real tokens, in raster order
        qp[idx], kp[idx], vp[idx] = q, k, v
        mask = o.sta_mask(cp, cp, gp, tile, window) & real[None, :]
        outp = o.masked_softmax_attention(qp, kp, vp, mask, 0.3)
        got = o.sta_attention_head(q, k, v, grid, tile, window, 0.3, pad=True)
        assert np.max(np.abs(outp[idx] - got)) < 1e-12


def pin_padding_is_noop_on_tile_multiples(o):
    grid, tile, window, d = (4, 8, 8), (2, 4, 4), (1, 3, 1), 8
    q, k, v = _rand_qkv(256, d, seed=31)
    a = o.sta_attention_head(q, k, v, grid, tile, window, 0.4)
    b = o.sta_attention_head(q, k, v, grid, tile, window, 0.4, pad=True)
    assert np.max(np.abs(a - b)) == 0.0
    assert o.attended_pairs_head(grid, tile, window) == o.attended_pairs_head(grid, tile, window, pad=True)


# ----------------------------------------------------------------------------- log-sum-exp and backward


def _masked_scores_torch(q, k, grid, tile, window, scale, pad=False):
    """Scaled scores with the brute-force mask (plain loops) applied, as a torch tensor."""
    mask = torch.from_numpy(_brute_mask(grid, tile, window, pad))
    s = scale * (torch.from_numpy(q) @ torch.from_numpy(k).T)
    return s.masked_fill(~mask, float("-inf")), mask


def pin_lse_matches_library(o):
    """Log-sum-exp over the brute-force window, by torch.logsumexp."""
    for grid, tile, window, d, pad in [((4, 8, 8), (2, 4, 4), (1, 3, 1), 8, False),
                                       ((3, 4, 6), (1, 2, 2), (2, 2, 3), 6, False),
                                       ((5, 7, 9), (2, 4, 4), (3, 3, 3), 4, True)]:
        L = int(np.prod(grid))
        q, k, _ = _rand_qkv(L, d, seed=3 * L + d)
        s, _ = _masked_scores_torch(q, k, grid, tile, window, 0.45, pad)
        want = torch.logsumexp(s, dim=1).numpy()
        got = o.sta_lse_head(q, k, grid, tile, window, 0.45, pad=pad)
        assert np.max(np.abs(got - want)) < 1e-12


def pin_lse_closed_forms(o):
    """q = 0 makes every allowed score zero, so lse_i = log(number of keys in the window)
    = log(Ntile * prod min(w, n)); adding one vector c to every key shifts row i's scores,
    and so its lse, by scale * q_i . c."""
    for grid, tile, window in [((4, 8, 8), (2, 4, 4), (1, 3, 5)), ((6, 4, 10), (2, 2, 2), (3, 1, 2))]:
        L, d, scale = int(np.prod(grid)), 5, 0.8
        n = [g // t for g, t in zip(grid, tile)]
        count = int(np.prod(tile)) * int(np.prod([min(w, m) for w, m in zip(window, n)]))
        q, k, _ = _rand_qkv(L, d, seed=L + 1)
        got = o.sta_lse_head(np.zeros_like(q), k, grid, tile, window, scale)
        assert np.max(np.abs(got - np.log(count))) < 1e-12
        c = np.linspace(-1.0, 1.5, d)
        shifted = o.sta_lse_head(q, k + c, grid, tile, window, scale)
        assert np.max(np.abs(shifted - o.sta_lse_head(q, k, grid, tile, window, scale) - scale * (q @ c))) < 1e-10


def _autograd_reference(q, k, v, do, mask, scale):
    """dq, dk, dv of scaled_dot_product_attention with a boolean mask, by torch autograd."""
    t = [torch.from_numpy(np.ascontiguousarray(x)).clone().requires_grad_(True) for x in (q, k, v)]
    out = torch.nn.functional.scaled_dot_product_attention(*[x[None, None] for x in t], attn_mask=mask[None, None],
                                                           scale=scale)[0, 0]
    out.backward(torch.from_numpy(np.ascontiguousarray(do)))
    return [x.grad.numpy() for x in t]


def pin_backward_equals_autograd(o):
    """Dense, per-tile and padded windows against torch autograd of masked SDPA."""
    for grid, tile, window, d, pad in [((4, 8, 8), (2, 4, 4), (3, 3, 3), 8, False),   # window = grid: dense
                                       ((4, 8, 8), (2, 4, 4), (1, 1, 1), 8, False),   # per tile
                                       ((3, 6, 8), (1, 2, 4), (1, 3, 1), 6, False),
                                       ((5, 7, 9), (2, 4, 4), (1, 3, 3), 4, True)]:
        L = int(np.prod(grid))
        q, k, v = _rand_qkv(L, d, seed=7 * L + d)
        do = _rand_qkv(L, d, seed=L)[0]
        mask = torch.from_numpy(_brute_mask(grid, tile, window, pad))
        want = _autograd_reference(q, k, v, do, mask, 0.6)
        got = o.sta_attention_backward_head(q, k, v, do, grid, tile, window, 0.6, pad=pad)
        for g, w in zip(got, want):
            assert np.max(np.abs(g - w)) < 1e-11


def pin_backward_finite_differences(o):
    """Central differences of sum(O * dO) through the (separately pinned) forward."""
    grid, tile, window, d, scale = (2, 4, 4), (1, 2, 2), (1, 3, 1), 4, 0.7
    L = 32
    q, k, v = _rand_qkv(L, d, seed=11)
    do = _rand_qkv(L, d, seed=12)[0]
    grads = o.sta_attention_backward_head(q, k, v, do, grid, tile, window, scale)
    rng = np.random.default_rng(13)
    h = 1e-6
    for which in range(3):
        for _ in range(8):
            i, j = int(rng.integers(L)), int(rng.integers(d))
            args = [q.copy(), k.copy(), v.copy()]
            args[which][i, j] += h
            fp = np.sum(o.sta_attention_head(*args, grid, tile, window, scale) * do)
            args[which][i, j] -= 2 * h
            fm = np.sum(o.sta_attention_head(*args, grid, tile, window, scale) * do)
            fd = (fp - fm) / (2 * h)
            assert abs(fd - grads[which][i, j]) < 1e-6 * max(1.0, abs(fd)), (which, i, j, fd, grads[which][i, j])


def pin_backward_closed_forms(o):
    """Rows of P sum to one, so the value gradients sum to the output gradients;
    rows of dS sum to zero, so the key gradients sum to zero."""
    grid, tile, window, d = (3, 8, 8), (1, 4, 4), (1, 1, 3), 8
    L = int(np.prod(grid))
    q, k, v = _rand_qkv(L, d, seed=21)
    do = _rand_qkv(L, d, seed=22)[0]
    dq, dk, dv = o.sta_attention_backward_head(q, k, v, do, grid, tile, window, 0.3)
    assert np.max(np.abs(dv.sum(axis=0) - do.sum(axis=0))) < 1e-10
    assert np.max(np.abs(dk.sum(axis=0))) < 1e-10


ALL_PINS = [
    pin_index_map_golden,
    pin_index_map_properties,
    pin_reorder_roundtrip,
    pin_window_golden,
    pin_mask_brute_force,
    pin_pair_counts,
    pin_dense_equals_library,
    pin_window_111_is_per_tile_attention,
    pin_uniform_softmax_mean,
    pin_permutation_invariance,
    pin_rows_normalised_and_hull,
    pin_sampled_rows_match_full,
    pin_padding_golden,
    pin_padding_brute_force,
    pin_padding_equals_explicit_padded_grid,
    pin_padding_is_noop_on_tile_multiples,
    pin_lse_matches_library,
    pin_lse_closed_forms,
    pin_backward_equals_autograd,
    pin_backward_finite_differences,
    pin_backward_closed_forms,
]
