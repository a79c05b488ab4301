"""Plain fp64 CPU oracle for the segment-over-cache attention path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product (the C-ABI library and its
Python binding in ``kv_cached_segment_b200``) imports, calls or links this
package.  It may be used by ``tests/``, by ``__graft_entry__.smoke()`` and by
``bench.py``'s CPU-baseline leg, nowhere else.

It shares no code with the CUDA path: only the seeded input generators of
``seeded_inputs`` serve both.  Every function is the plain definition of what
the path computes, written from the pages, in numpy float64; each cites the
passage it follows.  All functions are pinned by ``tests/test_oracle_pins.py``
against values and properties fixed by the pages and by mathematics.
"""
from .nomas_oracle import (  # noqa: F401
    bf16_bits_to_f64,
    video_positions,
    rope_frequencies,
    rope3d,
    kvcache_append,
    kvcache_select,
    attention,
    attention_rows,
    temporal_context_frame_indices,
    f32_to_bf16_bits,
    quantize_int8,
    dequantize_int8,
    dequantize_int8_f64,
    round_to_bf16_bits,
    key_tiles,
    block_sparse_attention,
    merge_partials,
)
