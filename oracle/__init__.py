"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Imported by ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs; never by the ``io_aware_softmax_b200`` package, which fails loudly when
its CUDA library is missing instead of falling back to anything here.
"""
from .attention import (  # noqa: F401
    MASK_CAUSAL, MASK_DOCUMENT_CAUSAL, MASK_SLIDING, MASK_NONE, MASK_SLIDING_CAUSAL,
    TILE_EMPTY, TILE_FULL, TILE_PARTIAL,
    attention, attention_backward, attention_head, attention_tiled_online, decode_paged, decode_splitkv, default_scale,
    document_ids, gather_paged, head_scores, merge_partials, softcap_scores, softmax_rows, split_bounds,
    tile_map, visible, visible_pairs,
)
