"""B200-native LSA (LongCat Sparse Attention) hot path.

The compute lives in ``liblsa.so`` (hand-written sm_100a CUDA behind the C ABI
declared in ``include/lsa.h``); ``kv_indexing_b200.lsa`` is its ctypes binding
and ``kv_indexing_b200.inputs`` draws seeded synthetic workloads.
"""
from . import inputs  # noqa: F401
from .lsa import (  # noqa: F401
    EXPORTS, LsaError, load, workspace_size, indexer_in, attn_in,
    lsa_index_flat, lsa_select_streaming, lsa_pool_pages, lsa_index_hier,
    lsa_sparse_attn, lsa_layer_group, lsa_device_status, lsa_pool_pages_e4m3, lsa_index_hier_e4m3,
    lsa_select_streaming_noalloc, lsa_index_compressed,
)
