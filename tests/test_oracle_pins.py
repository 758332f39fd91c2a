"""The CPU oracle against its pins, and the pins against planted mistakes.

Every pin must pass on the oracle as written.  Each mutant below plants one
plausible mistake in the oracle (on the CPU, inside this process) and at least
one pin must then fail: that is the evidence that the pins have teeth.
"""
import numpy as np
import pytest

import oracle.sta_oracle as O
import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(O)


def _mut_no_clamp(a, weff, ntiles):
    return a - weff // 2


def _mut_centre_up(a, weff, ntiles):
    return np.clip(a - (weff - 1) // 2, 0, np.asarray(ntiles) - weff)


def _mut_start_off_by_one(a, weff, ntiles):
    return np.clip(a - weff // 2 + 1, 0, np.asarray(ntiles) - weff)


def _mut_no_scale(q, k, v, mask, scale, return_p=False):
    return _orig_msa(q, k, v, mask, 1.0, return_p)


def _mut_softmax_axis0(q, k, v, mask, scale, return_p=False):
    s = scale * (np.asarray(q, float) @ np.asarray(k, float).T)
    s = np.where(mask, s, -np.inf)
    with np.errstate(invalid="ignore", divide="ignore"):
        s = s - s.max(axis=0, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=0, keepdims=True)
    p = np.nan_to_num(p)
    o = p @ np.asarray(v, float)
    return (o, p) if return_p else o


def _mut_keys_for_values(q, k, v, mask, scale, return_p=False):
    return _orig_msa(q, k, k, mask, scale, return_p)


def _mut_local_w_slowest(grid, tile):
    nT, nH, nW = O.tile_grid(grid, tile)
    tt, th, tw = tile
    c = O.raster_coords(grid)
    a = c // np.array(tile)
    r = c % np.array(tile)
    tile_id = (a[:, 0] * nH + a[:, 1]) * nW + a[:, 2]
    local = (r[:, 2] * th + r[:, 1]) * tt + r[:, 0]
    return tile_id * (tt * th * tw) + local


def _mut_tile_grid_hw_swapped(grid, tile):
    nT, nH, nW = O.tile_grid(grid, tile)
    tt, th, tw = tile
    c = O.raster_coords(grid)
    a = c // np.array(tile)
    r = c % np.array(tile)
    tile_id = (a[:, 0] * nW + a[:, 2]) * nH + a[:, 1]
    local = (r[:, 0] * th + r[:, 1]) * tw + r[:, 2]
    return tile_id * (tt * th * tw) + local


def _mut_coords_hw_swapped(grid):
    T, H, W = (int(x) for x in grid)
    n = np.arange(T * H * W, dtype=np.int64)
    return np.stack([n // (H * W), n % H, (n // H) % W], axis=1)


def _mut_mask_transposed(q_coords, k_coords, grid, tile, window, pad=False):
    return _orig_mask(k_coords, q_coords, grid, tile, window, pad).T


def _mut_mask_token_granular(q_coords, k_coords, grid, tile, window, pad=False):
    # token-wise sliding window: the window counted in tokens, not tiles
    return _orig_mask(q_coords, k_coords, grid, (1, 1, 1), window, pad)


def _mut_pad_floor(grid, tile, pad=False):
    # padded tile grid rounded down instead of up (edge tokens lose their tile)
    g, t = np.array([int(x) for x in grid]), np.array([int(x) for x in tile])
    if pad:
        return tuple(int(x) for x in np.maximum(g // t, 1))
    return _orig_tile_grid(grid, tile, pad)


def _mut_bwd_no_d_term(q, k, v, mask, scale, do):
    _, p = _orig_msa(q, k, v, mask, scale, return_p=True)
    dp = np.asarray(do, float) @ np.asarray(v, float).T
    ds = p * dp
    return scale * (ds @ np.asarray(k, float)), scale * (ds.T @ np.asarray(q, float)), p.T @ np.asarray(do, float)


def _mut_bwd_dq_unscaled(q, k, v, mask, scale, do):
    dq, dk, dv = _orig_bwd(q, k, v, mask, scale, do)
    return dq / scale, dk, dv


def _mut_bwd_dv_unnormalised(q, k, v, mask, scale, do):
    dq, dk, _ = _orig_bwd(q, k, v, mask, scale, do)
    s = scale * (np.asarray(q, float) @ np.asarray(k, float).T)
    e = np.exp(np.where(mask, s, -np.inf) - s.max(axis=1, keepdims=True))
    return dq, dk, e.T @ np.asarray(do, float)


def _mut_lse_base2(q, k, mask, scale):
    return _orig_lse(q, k, mask, scale) / np.log(2.0)


_orig_msa = O.masked_softmax_attention
_orig_bwd = O.masked_softmax_attention_backward
_orig_lse = O.masked_logsumexp
_orig_mask = O.sta_mask
_orig_tile_grid = O.tile_grid

MUTANTS = {
    "window_not_clamped": ("window_start", _mut_no_clamp),
    "even_window_centred_up": ("window_start", _mut_centre_up),
    "window_start_off_by_one": ("window_start", _mut_start_off_by_one),
    "scale_dropped": ("masked_softmax_attention", _mut_no_scale),
    "softmax_over_queries": ("masked_softmax_attention", _mut_softmax_axis0),
    "keys_used_as_values": ("masked_softmax_attention", _mut_keys_for_values),
    "tile_local_order_w_slowest": ("tiled_of_raster", _mut_local_w_slowest),
    "tile_grid_h_w_swapped": ("tiled_of_raster", _mut_tile_grid_hw_swapped),
    "raster_h_w_swapped": ("raster_coords", _mut_coords_hw_swapped),
    "mask_transposed": ("sta_mask", _mut_mask_transposed),
    "token_granular_window": ("sta_mask", _mut_mask_token_granular),
    "padded_tile_grid_rounded_down": ("tile_grid", _mut_pad_floor),
    "backward_without_row_term": ("masked_softmax_attention_backward", _mut_bwd_no_d_term),
    "backward_dq_unscaled": ("masked_softmax_attention_backward", _mut_bwd_dq_unscaled),
    "backward_dv_unnormalised": ("masked_softmax_attention_backward", _mut_bwd_dv_unnormalised),
    "logsumexp_in_base_2": ("masked_logsumexp", _mut_lse_base2),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(O)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin detects the planted mistake {name!r}"
