"""CPU oracle (float64) for exact split decode attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.  It shares no
code with the CUDA library.  See ``attention.py`` for the definitions and the
passages they follow.
"""
from .attention import (  # noqa: F401
    Partial,
    anchor_block_attention,
    anchor_visible_keys,
    attention_heads_cache,
    attention_one,
    attention_one_bf16_cache,
    bf16_to_f64,
    bifurcated_attention,
    chunk_partial,
    decode_attention,
    energy,
    finalize,
    gather_paged_sequence,
    merge,
    merge_shard_results,
    merge_tree,
    multi_query_attention,
    online_softmax,
    paged_decode_attention,
    paged_multi_query_attention,
    sequence_block,
    shard_bounds,
    split_attention,
    to_f64,
)
