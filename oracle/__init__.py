"""CPU oracle (test infrastructure only; never imported by the product path)."""

from .paged_attention import (ORACLE, PagedAttentionOracle, attend, copy_blocks,
                              decode, decode_one, gather, logical_pool, merge,
                              partial, physical_pool, swap_blocks, tile_offset,
                              write_kv)

__all__ = ["ORACLE", "PagedAttentionOracle", "attend", "copy_blocks", "decode",
           "decode_one", "gather", "logical_pool", "merge", "partial",
           "physical_pool", "swap_blocks", "tile_offset", "write_kv"]
