"""CPU oracle for Sliding Tile Attention forward (test infrastructure only).

Imported by the tests, the smoke check and the benchmark's CPU-baseline leg;
never by the product path.
"""
from .sta_oracle import (  # noqa: F401
    attended_flops,
    attended_pairs,
    attended_pairs_head,
    effective_window,
    masked_softmax_attention,
    raster_coords,
    reorder,
    sta_attention,
    sta_attention_head,
    sta_mask,
    tile_grid,
    tiled_of_raster,
    unorder,
    window_start,
)
