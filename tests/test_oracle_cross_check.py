"""The C++ oracle against the independent numpy/BLAS restatement, function by
function, and against itself at different thread counts (no GPU).

The two implementations share nothing but the definitions: the C++ one sums in
plain loops, the numpy one through BLAS. Float64 sums in another order can move
a float32 score by one unit in the last place, so scores are compared to one
ulp; everything decided from identical inputs (codes, selections, pooled keys,
recalled pages) must be identical.
"""
import numpy as np
import pytest

import oracle as O
from oracle import numpy_oracle as N
from kv_indexing_b200 import inputs as I


def _ulp_close(a, b):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    assert np.array_equal(np.isneginf(a), np.isneginf(b))
    fin = np.isfinite(a)
    gap = np.abs(a[fin].astype(np.float64) - b[fin].astype(np.float64))
    assert (gap <= np.spacing(np.abs(b[fin])).astype(np.float64)).all(), float(gap.max())


def test_codecs_agree():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 30, [0.0, -0.0, 448.0, 1e-9, np.inf]])
    x = x.astype(np.float32)
    assert np.array_equal(O.f32_to_bf16_rne(x), N.f32_to_bf16_rne(x))
    bits = np.arange(1 << 16, dtype=np.uint16)
    a, b = O.bf16_to_f64(bits), N.bf16_to_f64(bits)
    assert np.array_equal(a, b, equal_nan=True)
    codes = np.arange(256, dtype=np.uint8)
    assert np.array_equal(O.e4m3_to_f64(codes), N.e4m3_to_f64(codes), equal_nan=True)
    y = rng.standard_normal(20000) * 100
    assert np.array_equal(O.f64_to_e4m3_rne(y), N.f64_to_e4m3_rne(y))


@pytest.mark.parametrize("fp8", [False, True])
def test_flat_indexing_agrees(fp8):
    w = I.Workload(name="x", B=2, L=1024, T=5, H=8, d=64, k=96, sink=8, window=24, needles=10, fp8=fp8)
    x = I.make_indexer_inputs(w, 5)
    if fp8:
        args = (x["q_idx_fp8"], x["w"], x["k_idx_fp8"], x["seq_len"])
        kw = dict(fp8=True, q_scale=x["q_scale"], k_scale=x["k_scale"])
    else:
        args, kw = (x["q_idx"], x["w"], x["k_idx"], x["seq_len"]), {}
    sc_c, sc_n = O.indexer_scores(*args, **kw), N.indexer_scores(*args, **kw)
    _ulp_close(sc_c, sc_n)
    # the selection from one and the same score tensor must be identical
    assert np.array_equal(O.select_streaming(sc_n, x["seq_len"], w.T, w.k, w.sink, w.window),
                          N.select_streaming(sc_n, x["seq_len"], w.T, w.k, w.sink, w.window))


def test_selection_agrees_with_heavy_ties():
    rng = np.random.default_rng(9)
    sc = (rng.integers(0, 5, size=(3, 4, 700)) * 0.5).astype(np.float32)
    sc[0, :, 3::7] = -0.0
    sl = np.array([700, 333, 20], np.int32)
    for b in range(3):
        for t in range(4):
            sc[b, t, max(0, sl[b] - 4 + t + 1):] = -np.inf
    for k, s, win in [(64, 4, 8), (300, 0, 0), (16, 8, 8)]:
        assert np.array_equal(O.select_streaming(sc, sl, 4, k, s, win), N.select_streaming(sc, sl, 4, k, s, win))


def test_pooling_agrees():
    w = I.Workload(name="p", B=2, L=2048, T=1, H=4, d=64, k=64, sink=4, window=4, fp8=True)
    x = I.make_indexer_inputs(w, 2)
    sl = np.array([2048, 1000], np.int32)
    for P in (16, 64):
        assert np.array_equal(O.pool_pages(x["k_idx"], sl, P), N.pool_pages(x["k_idx"], sl, P))
        c1, s1 = O.pool_pages_e4m3(x["k_idx_fp8"], x["k_scale"], sl, P)
        c2, s2 = N.pool_pages_e4m3(x["k_idx_fp8"], x["k_scale"], sl, P)
        assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_hierarchical_indexing_agrees():
    w = I.Workload(name="h", B=2, L=4096, T=3, H=16, d=128, k=256, sink=16, window=64, needles=30, P=16, M=40,
                   fp8=True)
    x = I.make_indexer_inputs(w, 3)
    sl = np.array([4096, 2500], np.int32)
    pk = O.pool_pages(x["k_idx"], sl, w.P)
    kw = dict(P=w.P, M=w.M, budget=w.k, sink=w.sink, window=w.window)
    i1, p1 = O.index_hier(x["q_idx"], x["w"], x["k_idx"], pk, sl, **kw)
    i2, p2 = N.index_hier(x["q_idx"], x["w"], x["k_idx"], pk, sl, **kw)
    assert np.array_equal(i1, i2) and np.array_equal(p1, p2)
    pc, ps = O.pool_pages_e4m3(x["k_idx_fp8"], x["k_scale"], sl, w.P)
    e1 = O.index_hier_e4m3(x["q_idx_fp8"], x["q_scale"], x["w"], x["k_idx_fp8"], x["k_scale"], pc, ps, sl, **kw)
    e2 = N.index_hier_e4m3(x["q_idx_fp8"], x["q_scale"], x["w"], x["k_idx_fp8"], x["k_scale"], pc, ps, sl, **kw)
    assert np.array_equal(e1[0], e2[0]) and np.array_equal(e1[1], e2[1])
    for pos in (0, 15, 100, 1000, 4095):
        assert O.page_sets(pos, 16, 16, 64)[0] == N.page_sets(pos, 16, 16, 64)[0]
        assert O.page_sets(pos, 16, 16, 64)[1] == N.page_sets(pos, 16, 16, 64)[1]
        assert O.streaming_regions(pos, 16, 64) == N.streaming_regions(pos, 16, 64)


def test_compressed_entries_agree():
    w = I.Workload(name="c", B=2, L=4096, T=3, H=8, d=64, k=64, sink=4, window=12, needles=20, m=4)
    x = I.make_compressed_inputs(w, 4)
    x["seq_len"] = np.array([4096, 1234], np.int32)
    kw = dict(m=4, budget=w.k, sink=w.sink, window=w.window)
    i1, s1 = O.index_compressed(x["q_idx"], x["w"], x["entry_keys"], x["seq_len"], **kw)
    i2, s2 = N.index_compressed(x["q_idx"], x["w"], x["entry_keys"], x["seq_len"], **kw)
    _ulp_close(s1, s2)
    assert np.array_equal(i1, i2)


@pytest.mark.parametrize("mla", [False, True])
def test_attention_agrees(mla):
    w = I.Workload(name="a", B=2, L=512, T=2, H=4, d=64, k=80, sink=4, window=8, Hq=8,
                   d_qk=576 if mla else 64, d_v=512 if mla else 64, mla=mla)
    a = I.make_attn_inputs(w, 6)
    rng = np.random.default_rng(6)
    idx = rng.integers(-1, w.L, size=(w.B, w.T, w.k)).astype(np.int32)
    kw = dict(scale=0.11, d_v=w.d_v, kv=a.get("kv"), k=a.get("k"), v=a.get("v"))
    o1, l1 = O.sparse_attention(a["qa"], idx, None, **kw)
    o2, l2 = N.sparse_attention(a["qa"], idx, None, **kw)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-13) and np.allclose(l1, l2, rtol=1e-13)


def test_thread_count_does_not_change_results():
    w = I.Workload(name="t", B=3, L=20000, T=2, H=8, d=64, k=128, sink=8, window=16, needles=50)
    x = I.make_indexer_inputs(w, 8)
    outs = []
    for n in (1, 3, 0):
        O.set_threads(n)
        try:
            outs.append(O.index_flat(x["q_idx"], x["w"], x["k_idx"], x["seq_len"], budget=w.k, sink=w.sink,
                                     window=w.window))
        finally:
            O.set_threads(0)
    for idx, sc in outs[1:]:
        assert np.array_equal(idx, outs[0][0])
        assert np.array_equal(sc.view(np.uint32), outs[0][1].view(np.uint32))
