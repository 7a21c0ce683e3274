"""Hierarchical indexing on the GPU: page pooling (bit-exact), recall sets and
fine index sets vs the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I
from kv_indexing_b200 import lsa as L
from tests.parity import check_hier_rows, dev, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("P", [16, 64, 128])
def test_pool_pages_bit_exact(P):
    w = I.scaled(I.WORKLOADS["hier_decode_1m"], B=2, L=8192)
    x = I.make_indexer_inputs(w, 1)
    sl = np.array([8192, 8192 - 3 * P - 5], np.int32)            # second sequence ends mid-page
    pk = L.lsa_pool_pages(dev(x["k_idx"], "bf16"), dev(sl, "i32"), P)
    torch.cuda.synchronize()
    got = host(pk)
    ref = O.pool_pages(x["k_idx"], sl, P)
    for b in range(2):
        nf = int(sl[b]) // P
        assert np.array_equal(got[b, :nf], ref[b, :nf])
        assert (got[b, nf:] == 0).all()                          # untouched (zero-initialised)


def check_hier(w, x, seq_len, P, M, budget):
    q, k = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16")
    sl = dev(seq_len, "i32")
    pk = L.lsa_pool_pages(k, sl, P)
    B, T = x["q_idx"].shape[:2]
    pages = torch.empty((B, T, M), dtype=torch.int32, device="cuda")
    idx, _ = L.lsa_index_hier(q, dev(x["w"], "f32"), k, sl, pk, P, M, budget, pages_out=pages)
    torch.cuda.synchronize()
    L.lsa_device_status()
    gi, gp = host(idx), host(pages)
    n_full = int(seq_len.min()) // P
    assert np.array_equal(host(pk)[:, :n_full], O.pool_pages(x["k_idx"], seq_len, P)[:, :n_full])
    check_hier_rows(x, seq_len, P, M, budget, gi, gp, [(b, t) for b in range(B) for t in range(T)])
    return gi, gp


def test_hier_decode_small():
    w = I.scaled(I.WORKLOADS["hier_decode_1m"], B=2, L=32768, M=64)
    x = I.make_indexer_inputs(w, 2)
    check_hier(w, x, x["seq_len"], w.P, w.M, (w.k, w.sink, w.window))


def test_hier_ragged_lengths_and_small_pages():
    w = I.Workload(name="h", B=3, L=4096, T=2, H=64, d=128, k=512, sink=32, window=200, needles=40, P=16, M=48)
    x = I.make_indexer_inputs(w, 3)
    sl = np.array([4096, 3001, 700], np.int32)
    check_hier(w, x, sl, 16, 48, (w.k, w.sink, w.window))


def test_hier_full_recall_matches_flat():
    w = I.scaled(I.WORKLOADS["hier_decode_1m"], B=2, L=8192, M=128)      # M * P >= L
    x = I.make_indexer_inputs(w, 4)
    gi, _ = check_hier(w, x, x["seq_len"], w.P, w.M, (w.k, w.sink, w.window))
    fi = L.lsa_index_flat(dev(x["q_idx"], "bf16"), dev(x["w"], "f32"), dev(x["k_idx"], "bf16"),
                          dev(x["seq_len"], "i32"), (w.k, w.sink, w.window))
    torch.cuda.synchronize()
    assert np.array_equal(gi, host(fi))


@pytest.mark.parametrize("P", [16, 64])
def test_pool_pages_e4m3_bit_exact(P):
    w = I.scaled(I.WORKLOADS["hier_decode_1m"], B=2, L=8192, fp8=True)
    x = I.make_indexer_inputs(w, 5)
    sl = np.array([8192, 8192 - 5 * P - 3], np.int32)             # second sequence ends mid-page
    codes, scales = L.lsa_pool_pages_e4m3(dev(x["k_idx_fp8"], "e4m3"), dev(x["k_scale"], "f32"), dev(sl, "i32"), P)
    torch.cuda.synchronize()
    got_c, got_s = host(codes.view(torch.uint8)), host(scales)
    ref_c, ref_s = O.pool_pages_e4m3(x["k_idx_fp8"], x["k_scale"], sl, P)
    for b in range(2):
        nf = int(sl[b]) // P
        assert np.array_equal(got_c[b, :nf], ref_c[b, :nf])
        assert np.array_equal(got_s[b, :nf].view(np.uint32), ref_s[b, :nf].view(np.uint32))
        assert (got_c[b, nf:] == 0).all() and (got_s[b, nf:] == 1.0).all()   # untouched


def check_hier_e4m3(x, seq_len, P, M, budget):
    k8, ks = dev(x["k_idx_fp8"], "e4m3"), dev(x["k_scale"], "f32")
    sl = dev(seq_len, "i32")
    codes, scales = L.lsa_pool_pages_e4m3(k8, ks, sl, P)
    B, T = x["q_idx"].shape[:2]
    pages = torch.empty((B, T, M), dtype=torch.int32, device="cuda")
    idx, _ = L.lsa_index_hier_e4m3(dev(x["q_idx_fp8"], "e4m3"), dev(x["q_scale"], "f32"), dev(x["w"], "f32"), k8, ks,
                                   sl, codes, scales, P, M, budget, pages_out=pages)
    torch.cuda.synchronize()
    L.lsa_device_status()
    check_hier_rows(x, seq_len, P, M, budget, host(idx), host(pages), [(b, t) for b in range(B) for t in range(T)],
                    fp8=True)
    return host(idx)


def test_hier_e4m3_decode():
    w = I.scaled(I.WORKLOADS["hier_decode_1m"], B=2, L=65536, M=128, fp8=True)
    x = I.make_indexer_inputs(w, 6)
    check_hier_e4m3(x, x["seq_len"], w.P, w.M, (w.k, w.sink, w.window))


def test_hier_e4m3_ragged_small_pages_and_full_recall():
    w = I.Workload(name="h8", B=3, L=4096, T=2, H=64, d=128, k=512, sink=32, window=200, needles=40, P=16, M=48,
                   fp8=True)
    x = I.make_indexer_inputs(w, 7)
    check_hier_e4m3(x, np.array([4096, 3001, 700], np.int32), 16, 48, (w.k, w.sink, w.window))
    # M * P >= L: the recall holds every page, so the index rows are flat e4m3 indexing's
    w2 = I.scaled(I.WORKLOADS["hier_decode_1m"], B=2, L=8192, M=128, fp8=True)
    x2 = I.make_indexer_inputs(w2, 8)
    gi = check_hier_e4m3(x2, x2["seq_len"], w2.P, w2.M, (w2.k, w2.sink, w2.window))
    fi = L.lsa_index_flat(dev(x2["q_idx_fp8"], "e4m3"), dev(x2["w"], "f32"), dev(x2["k_idx_fp8"], "e4m3"),
                          dev(x2["seq_len"], "i32"), (w2.k, w2.sink, w2.window), q_scale=dev(x2["q_scale"], "f32"),
                          k_scale=dev(x2["k_scale"], "f32"))
    torch.cuda.synchronize()
    assert np.array_equal(gi, host(fi))
