"""Hierarchical indexing on the GPU: page pooling (bit-exact), recall sets and
fine index sets vs the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I
from kv_indexing_b200 import lsa as L
from tests.parity import check_index_row, dev, host, lead_count

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


def page_scores_oracle(x, pk, b, t, pos, P):
    n = (pos + 1) // P
    return O.indexer_scores_row(O.bf16_to_f64(x["q_idx"][b, t]), x["w"][b, t].astype(np.float64),
                                O.bf16_to_f64(pk[b, :n]), n)


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
    pk_o = O.pool_pages(x["k_idx"], seq_len, P)
    assert np.array_equal(host(pk)[:, :int(seq_len.min()) // P], pk_o[:, :int(seq_len.min()) // P])
    oi, op = O.index_hier(x["q_idx"], x["w"], x["k_idx"], pk_o, seq_len, P=P, M=M, budget=budget[0],
                          sink=budget[1], window=budget[2])
    kd = None
    for b in range(B):
        for t in range(T):
            pos = int(seq_len[b]) - T + t
            forced, E = O.page_sets(pos, P, budget[1], budget[2])
            psc = np.full(pk_o.shape[1], -np.inf, np.float32)
            psc[:(pos + 1) // P] = page_scores_oracle(x, pk_o, b, t, pos, P)
            g_pages = gp[b, t][gp[b, t] >= 0]
            o_pages = op[b, t][op[b, t] >= 0]
            assert set(forced) <= set(g_pages.tolist())
            gd = np.setdiff1d(g_pages, forced)
            od = np.setdiff1d(o_pages, forced)
            if gd.size and not np.array_equal(gd, od):
                tau = float(psc[od].min())
                for pgi in np.setdiff1d(np.union1d(gd, od), np.intersect1d(gd, od)):
                    assert abs(float(psc[pgi]) - tau) <= 1e-3 * abs(tau), "page recall differs beyond near-ties"
            # token level: valid top-D over the GPU's recalled pages, by oracle scores
            if kd is None or kd[0] != b:
                kd = (b, O.bf16_to_f64(x["k_idx"][b, :int(seq_len[b])]))
            _, _, c_rng = O.streaming_regions(pos, budget[1], budget[2])
            cands = np.arange(c_rng.start, c_rng.stop)
            cands = cands[np.isin(cands // P, g_pages)]
            tsc = np.full(int(seq_len[b]), -np.inf, np.float32)
            if cands.size:
                tsc[cands] = O.indexer_scores_row(O.bf16_to_f64(x["q_idx"][b, t]), x["w"][b, t].astype(np.float64),
                                                  kd[1][cands], cands.size)
            ref = oi[b, t] if np.array_equal(gd, od) else O.select_streaming_row(tsc, pos, *budget)
            check_index_row(gi[b, t], ref, tsc, lead_count(pos, budget[1], budget[2]))
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
