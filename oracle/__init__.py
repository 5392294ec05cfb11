"""CPU oracle for the hybrid compressed attention path (test infrastructure).

Plain numpy in float64.  Only the test suite, the package smoke check and the
bench's CPU-baseline leg may import this package; the CUDA library never
calls it and shares no code with it.
"""
from .formats import (e4m3_decode, e4m3_encode, e4m3_value_table, bf16_decode,
                      bf16_encode, e2m1_value_table, e2m1_decode, e2m1_encode, e8m0_decode,
                      mxfp4_pack, mxfp4_unpack, mxfp4_decode, mxfp4_quantize)
from .method import (n_entries, pool_positions, pool_entries, pool_entries_per_channel,
                     requantize, requantize_mxfp4,
                     scale_block,
                     indexer_scores, topk, attend, window_positions,
                     hybrid_attention, dequant_slots, ring_slots)
from .layer import (layer_compress, layer_indexer_topk, layer_attention,
                    layer_attention_dense_keys)

__all__ = [
    "e4m3_decode", "e4m3_encode", "e4m3_value_table", "bf16_decode", "bf16_encode",
    "e2m1_value_table", "e2m1_decode", "e2m1_encode", "e8m0_decode", "mxfp4_pack",
    "mxfp4_unpack", "mxfp4_decode", "mxfp4_quantize", "requantize_mxfp4",
    "n_entries", "pool_positions", "pool_entries", "pool_entries_per_channel", "requantize", "scale_block", "indexer_scores",
    "topk", "attend", "window_positions", "hybrid_attention", "dequant_slots",
    "ring_slots", "layer_compress", "layer_indexer_topk", "layer_attention",
    "layer_attention_dense_keys",
]
