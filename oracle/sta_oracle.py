"""Plain CPU oracle for Sliding Tile Attention (STA): forward, the forward's
per-row log-sum-exp, and the backward (gradients of q, k and v).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its Python binding) never calls it, and this module imports
nothing from that path.

What STA computes, as the sources state it:
  * "Fast Video Generation with Sliding Tile Attention" (arXiv 2502.04507),
    abstract: attention is restricted to a local 3D window that slides tile
    by tile instead of token by token.
  * Same paper, summary page, "Method details" section: the latent video is cut
    into non-overlapping spatio-temporal tiles, so attention inside a tile
    pair is dense; "Core innovation" section: blocks are either fully attended
    or skipped (no mixed blocks); "Technical contribution" section: each head
    has its own window size.
  * Same paper, review reply on input resolution: the tile is (6, 8, 8) and
    the latent dimensions must be multiples of the tile.
  * The window rule, for which the pages print no formula: a window of
    (wt, wh, ww) tiles around the query tile, its centre clamped so that it
    stays inside the tile grid (the plainest reading of a window that slides
    tile by tile over a bounded grid).

STA is exact softmax attention under a mask, so this oracle is the masked
definition written out in fp64 over raster-order tokens: no tiles are
reordered, nothing is blocked, and softmax is taken over the whole row.

Readings where the sources are silent (each also listed in the design notes):
  * windows are counted in tiles; a window wider than the tile grid is clamped
    to the grid, w' = min(w, n) per dimension;
  * the window start in each dimension is s = clamp(a - floor(w'/2), 0, n - w'),
    a being the query tile coordinate; for an even w' the window therefore
    reaches one tile further below the query tile than above it;
  * tokens are in raster order n = (t * H + h) * W + w; the tiled order used by
    the fast kernels (the index map below) is raster over the tile grid, then
    raster inside a tile.
"""
from __future__ import annotations

from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

Dim3 = Tuple[int, int, int]


def _dim3(x) -> Dim3:
    t = tuple(int(v) for v in x)
    if len(t) != 3:
        raise ValueError(f"expected three values, got {x!r}")
    return t  # type: ignore[return-value]


def raster_coords(grid: Sequence[int]) -> np.ndarray:
    """(t, h, w) of every token, in raster order n = (t * H + h) * W + w."""
    T, H, W = _dim3(grid)
    n = np.arange(T * H * W, dtype=np.int64)
    return np.stack([n // (H * W), (n // W) % H, n % W], axis=1)


def tile_grid(grid: Sequence[int], tile: Sequence[int], pad: bool = False) -> Dim3:
    """Number of tiles per dimension.

    Without padding the grid must be a multiple of the tile (review reply on input
    resolution: latents are (a*6, b*8, c*8)).  With padding (same reply, "padding
    with masking") the latent is conceptually padded up to the next tile multiple,
    so the tile grid is the ceiling; the pad tokens never take part as keys.
    """
    g, t = np.array(_dim3(grid)), np.array(_dim3(tile))
    if np.any(t <= 0) or np.any(g <= 0):
        raise ValueError(f"grid {tuple(g)} and tile {tuple(t)} must be positive")
    if pad:
        return _dim3(-(-g // t))
    if np.any(g % t != 0):
        raise ValueError(f"grid {tuple(g)} is not a positive multiple of tile {tuple(t)}")
    return _dim3(g // t)


def effective_window(window: Sequence[int], ntiles: Sequence[int]) -> np.ndarray:
    """w' = min(w, n) per dimension: a window wider than the grid covers the grid."""
    w = np.array(_dim3(window), dtype=np.int64)
    if np.any(w < 1):
        raise ValueError(f"window {tuple(w)} must be at least one tile per dimension")
    return np.minimum(w, np.array(_dim3(ntiles), dtype=np.int64))


def window_start(a: np.ndarray, weff: np.ndarray, ntiles: np.ndarray) -> np.ndarray:
    """First tile of the window of query tile ``a``, per dimension: the window is
    centred on the query tile and shifted back inside the grid at the edges."""
    return np.clip(a - weff // 2, 0, np.asarray(ntiles) - weff)


def sta_mask(q_coords: np.ndarray, k_coords: np.ndarray, grid, tile, window, pad: bool = False) -> np.ndarray:
    """Boolean mask[i, j]: the tile of key token j lies in the window of the tile
    of query token i.  Coordinates are token (t, h, w) triples of real tokens;
    with ``pad`` the tile grid is that of the latent padded to tile multiples."""
    ntiles = np.array(tile_grid(grid, tile, pad))
    tsz = np.array(_dim3(tile))
    weff = effective_window(window, ntiles)
    qa = np.asarray(q_coords) // tsz
    ka = np.asarray(k_coords) // tsz
    start = window_start(qa, weff, ntiles)
    mask = np.ones((qa.shape[0], ka.shape[0]), dtype=bool)
    for x in range(3):  # inside the window in every dimension
        mask &= (ka[None, :, x] >= start[:, None, x]) & (ka[None, :, x] < start[:, None, x] + weff[x])
    return mask


def masked_softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray,
                             scale: float, return_p: bool = False):
    """Textbook softmax(scale * q k^T) v with disallowed entries set to -inf, fp64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = scale * (q @ k.T)
    s = np.where(mask, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    o = p @ v
    return (o, p) if return_p else o


def sta_attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid, tile, window,
                       scale: float, rows: Optional[Iterable[int]] = None,
                       row_block: Optional[int] = None, pad: bool = False) -> np.ndarray:
    """STA forward of one (batch, head): q, k, v are [L, d] in raster order.

    Returns fp64 output rows for ``rows`` (all rows when None), in that order.
    Work is split into row blocks only to bound memory; each row's softmax runs
    over all L keys.  With ``pad`` the grid need not be a tile multiple: windows
    live on the padded tile grid and only the L real tokens are keys.
    """
    L = q.shape[0]
    coords = raster_coords(grid)
    if coords.shape[0] != L:
        raise ValueError("q rows do not match the grid")
    rows = np.arange(L) if rows is None else np.asarray(list(rows), dtype=np.int64)
    if row_block is None:
        row_block = int(min(512, max(16, (1 << 19) // L)))
    out = np.empty((rows.shape[0], v.shape[1]), dtype=np.float64)
    k64 = np.asarray(k, dtype=np.float64)
    v64 = np.asarray(v, dtype=np.float64)
    for r0 in range(0, rows.shape[0], row_block):
        sel = rows[r0:r0 + row_block]
        mask = sta_mask(coords[sel], coords, grid, tile, window, pad)
        out[r0:r0 + sel.shape[0]] = masked_softmax_attention(q[sel], k64, v64, mask, scale)
    return out


def masked_logsumexp(q: np.ndarray, k: np.ndarray, mask: np.ndarray, scale: float) -> np.ndarray:
    """Per row, log of the sum over allowed keys of exp(scale * q k^T), natural log,
    fp64; -inf for a row with no allowed key."""
    s = scale * (np.asarray(q, dtype=np.float64) @ np.asarray(k, dtype=np.float64).T)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1)
    safe = np.where(np.isfinite(m), m, 0.0)
    return safe + np.log(np.exp(s - safe[:, None]).sum(axis=1))


def sta_lse_head(q: np.ndarray, k: np.ndarray, grid, tile, window, scale: float,
                 rows: Optional[Iterable[int]] = None, pad: bool = False) -> np.ndarray:
    """Log-sum-exp of each query row's scaled scores over its window's keys (one
    (batch, head), raster order): the normaliser of the forward's softmax, which
    a backward pass reuses to rebuild P without a second row max."""
    L = q.shape[0]
    coords = raster_coords(grid)
    rows = np.arange(L) if rows is None else np.asarray(list(rows), dtype=np.int64)
    row_block = int(min(512, max(16, (1 << 19) // L)))
    out = np.empty(rows.shape[0], dtype=np.float64)
    for r0 in range(0, rows.shape[0], row_block):
        sel = rows[r0:r0 + row_block]
        out[r0:r0 + sel.shape[0]] = masked_logsumexp(q[sel], k, sta_mask(coords[sel], coords, grid, tile, window, pad),
                                                     scale)
    return out


def masked_softmax_attention_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray,
                                      scale: float, do: np.ndarray):
    """Gradients of O = softmax(scale * q k^T, masked) v with respect to q, k and v,
    given dO, by the chain rule written out in fp64:

        P = softmax(S),  dV = P^T dO,  dP = dO V^T,
        dS_ij = P_ij (dP_ij - D_i) with D_i = sum_j P_ij dP_ij (= dO_i . O_i),
        dQ = scale dS K,  dK = scale dS^T Q.

    Masked entries have P = 0 and so contribute nothing.  Returns (dq, dk, dv)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    _, p = masked_softmax_attention(q, k, v, mask, scale, return_p=True)
    dv = p.T @ do
    dp = do @ v.T
    dd = (p * dp).sum(axis=1, keepdims=True)
    ds = p * (dp - dd)
    return scale * (ds @ k), scale * (ds.T @ q), dv


def sta_attention_backward_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, do: np.ndarray, grid, tile,
                                window, scale: float, pad: bool = False):
    """STA backward of one (batch, head): q, k, v, dO are [L, d] in raster order.
    Returns fp64 (dq, dk, dv), each [L, d].  Query rows are taken in blocks only to
    bound memory; dk and dv add up every block's contribution."""
    L, d = q.shape
    coords = raster_coords(grid)
    if coords.shape[0] != L:
        raise ValueError("q rows do not match the grid")
    row_block = int(min(512, max(16, (1 << 19) // L)))
    dq = np.empty((L, d), dtype=np.float64)
    dk = np.zeros((L, d), dtype=np.float64)
    dv = np.zeros((L, v.shape[1]), dtype=np.float64)
    for r0 in range(0, L, row_block):
        sel = np.arange(r0, min(L, r0 + row_block))
        mask = sta_mask(coords[sel], coords, grid, tile, window, pad)
        gq, gk, gv = masked_softmax_attention_backward(q[sel], k, v, mask, scale, do[sel])
        dq[sel] = gq
        dk += gk
        dv += gv
    return dq, dk, dv


def sta_attention(q, k, v, grid, tile, windows, scale: float) -> np.ndarray:
    """STA forward over [B, heads, L, d] raster-order tensors; windows per head."""
    q = np.asarray(q, dtype=np.float64)
    B, Hn = q.shape[:2]
    if len(windows) != Hn:
        raise ValueError("one window per head is required")
    out = np.empty(q.shape, dtype=np.float64)
    for b in range(B):
        for h in range(Hn):
            out[b, h] = sta_attention_head(q[b, h], k[b, h], v[b, h], grid, tile, windows[h], scale)
    return out


def tiled_of_raster(grid, tile) -> np.ndarray:
    """Index map: raster token n -> its row in tiled order.

    Tiled order puts each tile's tokens in one contiguous run of Ntile rows
    (summary page, "Method details": tokens of a tile are contiguous).  Tiles
    follow raster order over the tile grid and tokens follow raster order
    inside a tile.
    """
    nT, nH, nW = tile_grid(grid, tile)
    tt, th, tw = _dim3(tile)
    c = raster_coords(grid)
    a = c // np.array([tt, th, tw])
    r = c % np.array([tt, th, tw])
    tile_id = (a[:, 0] * nH + a[:, 1]) * nW + a[:, 2]
    local = (r[:, 0] * th + r[:, 1]) * tw + r[:, 2]
    return tile_id * (tt * th * tw) + local


def reorder(x: np.ndarray, grid, tile) -> np.ndarray:
    """Raster -> tiled order along axis -2 (rows are tokens)."""
    m = tiled_of_raster(grid, tile)
    out = np.empty_like(x)
    out[..., m, :] = x
    return out


def unorder(x: np.ndarray, grid, tile) -> np.ndarray:
    """Tiled -> raster order along axis -2."""
    m = tiled_of_raster(grid, tile)
    return x[..., m, :]


def attended_pairs_head(grid, tile, window, pad: bool = False) -> int:
    """Number of (query, key) token pairs one head attends, counted by visiting
    every query tile and every key tile and testing window membership (with
    ``pad``, tiles count only their real tokens)."""
    ntiles = [int(x) for x in tile_grid(grid, tile, pad)]
    ntile_tokens = int(np.prod(_dim3(tile)))
    weff = [int(x) for x in effective_window(window, ntiles)]
    starts = []
    for dim in range(3):
        starts.append([int(window_start(np.int64(a), np.int64(weff[dim]), np.int64(ntiles[dim])))
                       for a in range(ntiles[dim])])
    total = 0
    for at in range(ntiles[0]):
        for ah in range(ntiles[1]):
            for aw in range(ntiles[2]):
                s = (starts[0][at], starts[1][ah], starts[2][aw])
                n_key_tiles = 0
                for kt in range(ntiles[0]):
                    for kh in range(ntiles[1]):
                        for kw in range(ntiles[2]):
                            if (s[0] <= kt < s[0] + weff[0] and s[1] <= kh < s[1] + weff[1]
                                    and s[2] <= kw < s[2] + weff[2]):
                                n_key_tiles += 1
                if not pad:
                    total += ntile_tokens * ntile_tokens * n_key_tiles
                else:
                    qn = _real_tokens_in_tile(grid, tile, (at, ah, aw))
                    kn = 0
                    for kt in range(s[0], s[0] + weff[0]):
                        for kh in range(s[1], s[1] + weff[1]):
                            for kw in range(s[2], s[2] + weff[2]):
                                kn += _real_tokens_in_tile(grid, tile, (kt, kh, kw))
                    total += qn * kn
    return int(total)


def _real_tokens_in_tile(grid, tile, a) -> int:
    """Real (not pad) tokens of tile ``a`` of the padded tile grid."""
    n = 1
    for x in range(3):
        lo = a[x] * tile[x]
        n *= max(0, min(grid[x], lo + tile[x]) - lo)
    return n


def attended_pairs(batch: int, grid, tile, windows, pad: bool = False) -> int:
    return int(batch) * sum(attended_pairs_head(grid, tile, w, pad) for w in windows)


def attended_flops(batch: int, d: int, grid, tile, windows) -> int:
    """4 * d FLOPs per attended pair: 2d for q.k, 2d for p * v."""
    return 4 * int(d) * attended_pairs(batch, grid, tile, windows)
