"""CPU oracle for the LSA hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may
import this package. The product path never does, and shares no code with it.
"""
from .lsa_oracle import *  # noqa: F401,F403
from .lsa_oracle import (  # noqa: F401
    bf16_to_f64, f32_to_bf16_rne, e4m3_to_f64, indexer_scores_row, indexer_scores,
    streaming_regions, top_by_score, select_streaming_row, select_streaming,
    index_flat, pool_pages, page_sets, index_hier_row, index_hier,
    sparse_attention_row, sparse_attention, layer_group, entry_position, index_compressed,
    f64_to_e4m3_rne, pool_pages_e4m3, index_hier_e4m3,
)
