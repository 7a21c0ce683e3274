"""The algorithmic work the bench divides by (roofline denominators), checked
against figures worked out by hand from the workloads' shapes."""
import bench
from kv_indexing_b200 import inputs as I


def test_flat_decode_indexer_bytes():
    # 8 queries x (keys 131072 x 128 x 2 B + q 64 x 128 x 2 B + w 64 x 4 B)
    w = I.WORKLOADS["flat_decode_128k"]
    assert bench.indexer_bytes_per_query(w) * w.B == 8 * (33554432 + 16384 + 256) == 268568576
    # e4m3 keys: one byte per element plus a 4-byte scale per key; q codes and scales per head
    assert bench.indexer_bytes_per_query(w, fp8=True) == 131072 * (128 + 4) + 64 * (128 + 4) + 64 * 4


def test_flat_decode_1m_indexer_bytes():
    w = I.WORKLOADS["flat_decode_1m"]
    assert bench.indexer_bytes_per_query(w) * w.B == 2 * (1048576 * 256 + 16384 + 256)


def test_attention_bytes():
    # 2048 gathered 576-wide latent rows (bf16) + q 128 x 576 + o 128 x 512, per query
    w = I.WORKLOADS["flat_decode_128k"]
    assert bench.attention_bytes_per_query(w) == 2359296 + 147456 + 131072
    assert bench.attention_bytes_per_query(w) * w.B == 21102592
    # e4m3 cache: 576 code bytes + a 4-byte scale per gathered row
    assert bench.attention_bytes_per_query(w, kv8=True) == 2048 * 580 + 147456 + 131072


def test_hierarchical_index_bytes():
    # 16384 page keys + 256 recalled pages x 64 tokens, 256 B each, + q + w
    w = I.WORKLOADS["hier_decode_1m"]
    assert bench.hier_index_bytes_per_query(w) == 4194304 + 4194304 + 16384 + 256
    assert bench.hier_index_bytes_per_query(w, fp8=True) == (16384 + 16384) * 132 + 64 * 132 + 256


def test_prefill_indexer_flops():
    # visible (query, key) pairs of the causal chunk at 61440..65535: sum of (pos + 1)
    w = I.WORKLOADS["prefill_64k"]
    pairs = (61441 + 65536) * 4096 // 2
    assert pairs == 260048896
    assert bench.prefill_indexer_flops(w) == 2.0 * 64 * 128 * pairs == 4260641112064.0
