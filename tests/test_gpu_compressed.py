"""Indexing over compressed entries on the GPU vs the oracle: entry scores,
entry index sets, the selection's entry position, and attention over the
chosen compressed latent entries."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I
from kv_indexing_b200 import lsa as L
from tests.parity import (accumulation_scale, assert_attention_close, assert_scores_close, check_index_row, dev,
                          host, same_rows)

pytestmark = pytest.mark.gpu


def run_gpu(x, m, budget, sl_np, fp8=False):
    if fp8:
        q, ek = dev(x["q_idx_fp8"], "e4m3"), dev(x["entry_keys_fp8"], "e4m3")
        qs, ks = dev(x["q_scale"], "f32"), dev(x["k_scale"], "f32")
    else:
        q, ek = dev(x["q_idx"], "bf16"), dev(x["entry_keys"], "bf16")
        qs = ks = None
    B, T = x["q_idx"].shape[:2]
    n_e = x["entry_keys"].shape[1]
    scores = torch.empty((B, T, n_e), dtype=torch.float32, device="cuda")
    idx = L.lsa_index_compressed(q, dev(x["w"], "f32"), ek, dev(sl_np, "i32"), m, budget, q_scale=qs, k_scale=ks,
                                 scores_out=scores)
    torch.cuda.synchronize()
    L.lsa_device_status()
    return host(idx), host(scores)


def check(x, m, budget, sl_np, fp8=False):
    gi, gs = run_gpu(x, m, budget, sl_np, fp8)
    kw = dict(fp8=True, q_scale=x["q_scale"], k_scale=x["k_scale"]) if fp8 else {}
    q = x["q_idx_fp8"] if fp8 else x["q_idx"]
    ek = x["entry_keys_fp8"] if fp8 else x["entry_keys"]
    oi, os_ = O.index_compressed(q, x["w"], ek, sl_np, m=m, budget=budget[0], sink=budget[1], window=budget[2],
                                 **kw)
    assert_scores_close(gs, os_, accumulation_scale(q, x["w"], ek, **kw))
    B, T = q.shape[:2]
    for b in range(B):
        for t in range(T):
            pe = O.entry_position(int(sl_np[b]) - T + t, m)
            if pe < 0:
                assert (gi[b, t] == -1).all()
                continue
            check_index_row(gi[b, t], oi[b, t], os_[b, t], pe, budget[1], budget[2])
    return gi


@pytest.mark.parametrize("m", [4, 16])
def test_compressed_decode(m):
    w = I.scaled(I.WORKLOADS["compressed_decode_1m"], B=3, L=4096 * m, m=m)
    x = I.make_compressed_inputs(w, 1)
    sl = np.array([w.L, w.L - 3, w.L - 7 * m - 1], np.int32)   # ragged: partial trailing entries
    check(x, m, (w.k, w.sink, w.window), sl)


def test_compressed_fp8_entry_keys():
    w = I.scaled(I.WORKLOADS["compressed_decode_1m"], B=2, L=16384)
    x = I.make_compressed_inputs(w, 2)
    check(x, w.m, (w.k, w.sink, w.window), np.array([16384, 9001], np.int32), fp8=True)


def test_compressed_many_queries_and_empty_rows():
    """T = 160 queries at tokens 40 .. 199 with m = 128: the 87 queries before
    token 127 see no complete entry (all -1), the later ones entry 0 only."""
    w = I.scaled(I.WORKLOADS["compressed_decode_1m"], B=1, L=16384, T=160, k=8, sink=1, window=1,
                 needle_frac=0.0, m=128)
    x = I.make_compressed_inputs(w, 3)
    gi = check(x, 128, (8, 1, 1), np.array([200], np.int32))
    assert (gi[0, :, 0] == -1).sum() == 87
    assert (gi[0, 87:, 0] == 0).all() and (gi[0, :, 1:] == -1).all()


def test_compressed_entry_size_one_equals_flat():
    w = I.scaled(I.WORKLOADS["flat_decode_128k"], B=2, L=8192, T=4)
    x = I.make_indexer_inputs(w, 4)
    q, k, ww, sl = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16"), dev(x["w"], "f32"), dev(x["seq_len"], "i32")
    budget = (w.k, w.sink, w.window)
    a = L.lsa_index_compressed(q, ww, k, sl, 1, budget)
    b = L.lsa_index_flat(q, ww, k, sl, budget)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_compressed_decode_then_attention_over_entries():
    """The workflow: choose entries, then attend to the chosen compressed
    latent entries (with the streaming-prefix promise, in entry units)."""
    w = I.scaled(I.WORKLOADS["compressed_decode_1m"], B=2, L=32768)
    x = I.make_compressed_inputs(w, 5)
    ew = I.entry_workload(w)
    a = I.make_attn_inputs(ew, 5)
    m = w.m
    sl_np = np.array([w.L, w.L - 2 * m], np.int32)
    budget = (w.k, w.sink, w.window)
    idx = L.lsa_index_compressed(dev(x["q_idx"], "bf16"), dev(x["w"], "f32"), dev(x["entry_keys"], "bf16"),
                                 dev(sl_np, "i32"), m, budget)
    sl_e = dev(sl_np // m, "i32")   # decode: the query's entry position is seq_len // m - 1
    out, _ = L.lsa_sparse_attn(dev(a["qa"], "bf16"), idx, sl_e, w.scale, kv=dev(a["kv"], "bf16"), d_v=w.d_v,
                               stream_budget=budget)
    torch.cuda.synchronize()
    L.lsa_device_status()
    gi = host(idx)
    oi, os_ = O.index_compressed(x["q_idx"], x["w"], x["entry_keys"], sl_np, m=m, budget=w.k, sink=w.sink,
                                 window=w.window)
    for b in range(w.B):
        check_index_row(gi[b, 0], oi[b, 0], os_[b, 0], O.entry_position(int(sl_np[b]) - 1, m), w.sink, w.window)
    rows = same_rows(gi, oi)
    assert rows, "no index row equals the oracle's"
    o_ref, _ = O.sparse_attention_rows(a["qa"], oi, rows, scale=w.scale, d_v=w.d_v, kv=a["kv"])
    g = O.bf16_to_f64(host(out))
    assert_attention_close(np.stack([g[b, t] for b, t in rows]), o_ref)
