"""CPU oracle of the LiteAttention forward pass (test infrastructure; never used by the product path)."""

from .lite_attention import (  # noqa: F401
    ForwardResult,
    QTileResult,
    attend_query_tile,
    dense_attention,
    geometry,
    is_skipped,
    lite_attention_forward,
    live_flop,
    lse_merge,
    range_tiles,
    live_key_tiles,
    mask_to_list,
    mask_to_ranges,
    schedule_order,
    tile_for_head_dim,
)
