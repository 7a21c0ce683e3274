"""Streaming top-k on the GPU vs the oracle, given the oracle's own scores:
bit-exact index rows (sink, window, dynamic ascending, -1 padding)."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I
from kv_indexing_b200 import lsa as L
from tests.parity import dev, host

pytestmark = pytest.mark.gpu


def run_select(scores, seq_len, T, budget):
    idx = L.lsa_select_streaming(dev(scores, "f32"), dev(seq_len, "i32"), budget)
    torch.cuda.synchronize()
    L.lsa_device_status()
    return host(idx)


def oracle_scores(w, seed, rows=None):
    x = I.make_indexer_inputs(w, seed)
    return O.indexer_scores(x["q_idx"], x["w"], x["k_idx"], x["seq_len"], rows=rows), x["seq_len"]


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_select_tiny_workload_bit_exact(seed):
    w = I.WORKLOADS["tiny_l2k"]
    sc, sl = oracle_scores(w, seed)
    budget = (w.k, w.sink, w.window)
    got = run_select(sc, sl, w.T, budget)
    ref = O.select_streaming(sc, sl, w.T, *budget)
    assert np.array_equal(got, ref)


def test_select_heavy_ties_negative_zero_and_short_rows():
    rng = np.random.default_rng(5)
    B, T, L_max = 3, 7, 3000
    sc = (rng.integers(0, 6, size=(B, T, L_max)) * 0.5).astype(np.float32)
    sc[rng.random(sc.shape) < 0.05] = -0.0
    sl = np.array([3000, 700, 40], np.int32)
    for t in range(T):                       # invisible slots carry -inf, like the indexer writes
        for b in range(B):
            sc[b, t, sl[b] - T + t + 1:] = -np.inf
    for budget in [(256, 64, 64), (64, 0, 0), (100, 20, 0), (50, 0, 50), (8, 3, 5)]:
        got = run_select(sc, sl, T, budget)
        ref = O.select_streaming(sc, sl, T, *budget)
        assert np.array_equal(got, ref), budget


def test_select_negative_scores_and_empty_rows():
    rng = np.random.default_rng(6)
    B, T, L_max = 2, 4, 512
    sc = rng.standard_normal((B, T, L_max)).astype(np.float32) * 100
    sl = np.array([2, 512], np.int32)        # b=0: queries 0,1 have pos < 0
    for b in range(B):
        for t in range(T):
            sc[b, t, max(0, sl[b] - T + t + 1):] = -np.inf
    got = run_select(sc, sl, T, (64, 4, 8))
    ref = O.select_streaming(sc, sl, T, 64, 4, 8)
    assert np.array_equal(got, ref)
    assert (got[0, 0] == -1).all() and (got[0, 1] == -1).all()


@pytest.mark.parametrize("B,L_max,ties", [(8, 131072, True), (3, 150001, True), (4, 262144, True),
                                          (2, 262144, False), (3, 393216, True), (2, 1 << 20, True)])
def test_select_long_rows_all_launch_paths(B, L_max, ties):
    # up to 128K slots: one cluster per row, 32 keys per thread; up to 256K: 64
    # keys per thread; 384K rows: the grid-cooperative launch (rows x CTAs fit
    # the GPU at once); 1M rows: per-segment candidates + merge. The tie block
    # overflows the boundary lists (exact radix rounds); without it the
    # window histogram decides.
    rng = np.random.default_rng(L_max)
    sc = rng.standard_normal((B, 1, L_max)).astype(np.float32)
    sc = np.abs(sc) + np.float32(3.0)
    if ties:
        sc[:, :, rng.integers(0, L_max, size=4000)] = np.float32(9.5)     # a block of exact ties
    sl = np.full((B,), L_max, np.int32)
    got = run_select(sc, sl, 1, (2048, 64, 960))
    ref = O.select_streaming(sc, sl, 1, 2048, 64, 960)
    assert np.array_equal(got, ref)


def _filter_rows(B, L_max, seq_len, kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "all_equal":                    # every candidate ties: the lowest slots win
        sc = np.full((B, 1, L_max), 2.5, np.float32)
    elif kind == "tie_block":                  # a block of exact ties straddles the threshold
        sc = (np.abs(rng.standard_normal((B, 1, L_max))) + 3.0).astype(np.float32)
        sc[:, :, rng.integers(0, L_max, size=3000)] = np.float32(5.25)
    elif kind == "holes":                      # -inf holes (not candidates) and -0
        sc = rng.standard_normal((B, 1, L_max)).astype(np.float32)
        sc[rng.random(sc.shape) < 0.3] = -np.inf
        sc[rng.random(sc.shape) < 0.01] = -0.0
    else:                                      # plain normal scores
        sc = rng.standard_normal((B, 1, L_max)).astype(np.float32)
    for b in range(B):
        sc[b, 0, seq_len[b]:] = -np.inf
    return sc


@pytest.mark.parametrize("kind", ["normal", "all_equal", "tie_block", "holes"])
def test_select_filter_launch_bit_exact(kind):
    # rows longer than a cluster holds and than the grid launch takes: the filter
    # launch (group-maximum bound, per-warp kept runs, last-CTA finish)
    B, L_max = 2, 1 << 20
    sl = np.array([L_max, 700001], np.int32)
    assert L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=B, T=1, L_max=L_max) > 0
    sc = _filter_rows(B, L_max, sl, kind, 7)
    for budget in [(2048, 64, 960), (300, 0, 0), (4096, 16, 16)]:
        got = run_select(sc, sl, 1, budget)
        assert np.array_equal(got, O.select_streaming(sc, sl, 1, *budget)), (kind, budget)


def test_select_filter_launch_short_and_empty_rows():
    B, L_max = 4, 600000
    sl = np.array([600000, 3000, 0, 599999], np.int32)   # a row shorter than the budget and an empty one
    sc = _filter_rows(B, L_max, sl, "normal", 8)
    got = run_select(sc, sl, 1, (2048, 64, 960))
    assert np.array_equal(got, O.select_streaming(sc, sl, 1, 2048, 64, 960))
    assert (got[2] == -1).all()


@pytest.mark.parametrize("L_max", [16384, 30000, 65536, 100000])
def test_select_cluster_keys_per_thread_variants_bit_exact(L_max):
    # two rows: the cluster of up to 8 CTAs per row holds 4, 8, 16 or 32 keys per
    # thread depending on the row length (the hierarchical selections' shapes)
    rng = np.random.default_rng(L_max)
    B = 2
    sl = np.array([L_max, L_max * 3 // 4], np.int32)
    sc = (rng.integers(0, 50, size=(B, 1, L_max)) * 0.125).astype(np.float32)   # many ties
    for b in range(B):
        sc[b, 0, sl[b]:] = -np.inf
    for budget in [(2048, 64, 960), (256, 0, 0), (1024, 8, 100)]:
        got = run_select(sc, sl, 1, budget)
        assert np.array_equal(got, O.select_streaming(sc, sl, 1, *budget)), budget
