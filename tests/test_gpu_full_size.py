"""GPU vs oracle at the workloads' own sizes, in the launch configuration the
benchmark times.

- flat decode, 8 x 131072 cached tokens, H_I=64, d_I=128, k=2048 (sink 64,
  window 960): scores of every row, every index row, attention of every row;
- flat prefill, one sequence of 65536 tokens, 4096 causal queries at positions
  61440..65535: scores and index rows on a stride of query rows, bf16 and e4m3;
- hierarchical decode, 2 x 1048576 tokens, P=64, M=256: page keys (bit-exact),
  recalled pages and index rows of both queries;
- cross-layer group, 4 x 262144, two MLA layers, hierarchical and flat: index
  rows and both layers' attention.

Every input is drawn by kv_indexing_b200.inputs with the workload's shapes;
the oracle reads the same bytes. Tolerances are the ones every parity test
uses (tests/parity.py)."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I
from kv_indexing_b200 import lsa as L
from tests.parity import (accumulation_scale_rows, assert_attention_close, assert_scores_close, check_hier_rows,
                          check_index_row, dev, host, same_rows)

pytestmark = pytest.mark.gpu


def budget_of(w):
    return (w.k, w.sink, w.window)


def test_flat_decode_128k_full_size():
    w = I.WORKLOADS["flat_decode_128k"]
    x = I.make_indexer_inputs(w, 1)
    a = I.make_attn_inputs(w, 1)
    budget = budget_of(w)
    q, k, ww, sl = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16"), dev(x["w"], "f32"), dev(x["seq_len"], "i32")
    scores = torch.empty((w.B, 1, w.L), dtype=torch.float32, device="cuda")
    gi = host(L.lsa_index_flat(q, ww, k, sl, budget, scores_out=scores))
    torch.cuda.synchronize()
    L.lsa_device_status()
    rows = [(b, 0) for b in range(w.B)]
    os_ = O.indexer_scores(x["q_idx"], x["w"], x["k_idx"], x["seq_len"])
    assert_scores_close(host(scores)[:, 0], os_[:, 0],
                        accumulation_scale_rows(x["q_idx"], x["w"], x["k_idx"], rows))
    oi = O.select_streaming(os_, x["seq_len"], 1, *budget)
    for b in range(w.B):
        check_index_row(gi[b, 0], oi[b, 0], os_[b, 0], w.L - 1, w.sink, w.window)
    # selection alone, given the oracle's scores: bit-exact
    assert np.array_equal(host(L.lsa_select_streaming(dev(os_, "f32"), sl, budget)), oi)
    # attention over the oracle's index set, with the streaming-prefix promise
    # the decode step uses
    out, _ = L.lsa_sparse_attn(dev(a["qa"], "bf16"), dev(oi, "i32"), sl, w.scale, kv=dev(a["kv"], "bf16"),
                               d_v=w.d_v, stream_budget=budget)
    torch.cuda.synchronize()
    L.lsa_device_status()
    o_ref, _ = O.sparse_attention(a["qa"], oi, x["seq_len"], scale=w.scale, d_v=w.d_v, kv=a["kv"])
    assert_attention_close(O.bf16_to_f64(host(out)), o_ref)


def test_flat_decode_1m_full_size_fused_selection():
    # 2 x 1M: the indexer writes the selection's group maxima beside the scores
    # (fused scoring + selection); its index rows must equal the oracle's, and
    # bit for bit the selection over the same scores without the fused summaries
    w = I.WORKLOADS["flat_decode_1m"]
    x = I.make_indexer_inputs(w, 1)
    budget = budget_of(w)
    q, k, ww, sl = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16"), dev(x["w"], "f32"), dev(x["seq_len"], "i32")
    scores = torch.empty((w.B, 1, w.L), dtype=torch.float32, device="cuda")
    gi = host(L.lsa_index_flat(q, ww, k, sl, budget, scores_out=scores))   # scores out: the selection reads them
    idx_ws = L.lsa_index_flat(q, ww, k, sl, budget)                          # scores in the workspace
    sel = L.lsa_select_streaming(scores, sl, budget)
    torch.cuda.synchronize()
    L.lsa_device_status()
    assert np.array_equal(gi, host(idx_ws))
    assert np.array_equal(gi, host(sel))
    rows = [(b, 0) for b in range(w.B)]
    os_ = O.indexer_scores_rows(x["q_idx"], x["w"], x["k_idx"], x["seq_len"], rows)
    for b in range(w.B):
        check_index_row(gi[b, 0], O.select_streaming_row(os_[b], w.L - 1, *budget), os_[b], w.L - 1, w.sink,
                        w.window)


@pytest.mark.parametrize("fp8", [False, True])
def test_prefill_64k_full_size_strided_rows(fp8):
    w = I.WORKLOADS["prefill_64k"]
    x = I.make_indexer_inputs(w, 1)
    budget = budget_of(w)
    if fp8:
        qn, kn = x["q_idx_fp8"], x["k_idx_fp8"]
        q, k = dev(qn, "e4m3"), dev(kn, "e4m3")
        qs, ks = dev(x["q_scale"], "f32"), dev(x["k_scale"], "f32")
        kw = dict(fp8=True, q_scale=x["q_scale"], k_scale=x["k_scale"])
    else:
        qn, kn = x["q_idx"], x["k_idx"]
        q, k = dev(qn, "bf16"), dev(kn, "bf16")
        qs = ks = None
        kw = {}
    sl = dev(x["seq_len"], "i32")
    scores = torch.empty((1, w.T, w.L), dtype=torch.float32, device="cuda")
    idx = L.lsa_index_flat(q, dev(x["w"], "f32"), k, sl, budget, q_scale=qs, k_scale=ks, scores_out=scores)
    torch.cuda.synchronize()
    L.lsa_device_status()
    ts = list(range(0, w.T, 257)) + [w.T - 1]            # first, last and a stride across every tile row
    rows = [(0, t) for t in ts]
    gs = host(scores[0, ts])
    gi = host(idx[0, ts])
    os_ = O.indexer_scores_rows(qn, x["w"], kn, x["seq_len"], rows, **kw)
    assert_scores_close(gs, os_, accumulation_scale_rows(qn, x["w"], kn, rows, **kw))
    for i, t in enumerate(ts):
        pos = w.L - w.T + t
        oi = O.select_streaming_row(os_[i], pos, *budget)
        check_index_row(gi[i], oi, os_[i], pos, w.sink, w.window)


def test_hier_decode_1m_full_size():
    w = I.WORKLOADS["hier_decode_1m"]
    x = I.make_indexer_inputs(w, 1)
    budget = budget_of(w)
    q, k, ww, sl = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16"), dev(x["w"], "f32"), dev(x["seq_len"], "i32")
    pk = L.lsa_pool_pages(k, sl, w.P)
    pages = torch.empty((w.B, 1, w.M), dtype=torch.int32, device="cuda")
    idx, _ = L.lsa_index_hier(q, ww, k, sl, pk, w.P, w.M, budget, pages_out=pages)
    torch.cuda.synchronize()
    L.lsa_device_status()
    assert np.array_equal(host(pk), O.pool_pages(x["k_idx"], x["seq_len"], w.P))
    check_hier_rows(x, x["seq_len"], w.P, w.M, budget, host(idx), host(pages), [(b, 0) for b in range(w.B)])


@pytest.fixture(scope="module")
def group_inputs():
    w = I.WORKLOADS["cli_group_256k"]
    return w, I.make_indexer_inputs(w, 1), [I.make_attn_inputs(w, 1, layer=i) for i in range(w.n_layers)]


@pytest.mark.parametrize("hier", [True, False])
def test_cli_group_256k_full_size(group_inputs, hier):
    w, x, lnps = group_inputs
    budget = budget_of(w)
    q, k, ww, sl = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16"), dev(x["w"], "f32"), dev(x["seq_len"], "i32")
    layers = [{"q": dev(l["qa"], "bf16"), "kv": dev(l["kv"], "bf16"), "scale": w.scale, "d_v": w.d_v} for l in lnps]
    P, M = (w.P, w.M) if hier else (0, 0)
    pk = L.lsa_pool_pages(k, sl, w.P) if hier else None
    idx, outs = L.lsa_layer_group(q, ww, k, sl, budget, layers, P=P, M=M, page_keys=pk)
    torch.cuda.synchronize()
    L.lsa_device_status()
    gi = host(idx)
    rows = [(b, 0) for b in range(w.B)]
    if hier:
        pages = torch.empty((w.B, 1, w.M), dtype=torch.int32, device="cuda")
        gi_single, _ = L.lsa_index_hier(q, ww, k, sl, pk, w.P, w.M, budget, pages_out=pages)
        torch.cuda.synchronize()
        assert np.array_equal(gi, host(gi_single))          # the group's index set is the single call's
        oi = check_hier_rows(x, x["seq_len"], w.P, w.M, budget, gi, host(pages), rows)
    else:
        os_ = O.indexer_scores(x["q_idx"], x["w"], x["k_idx"], x["seq_len"])
        oi = O.select_streaming(os_, x["seq_len"], 1, *budget)
        for b in range(w.B):
            check_index_row(gi[b, 0], oi[b, 0], os_[b, 0], w.L - 1, w.sink, w.window)
    cmp = same_rows(gi, oi)
    assert len(cmp) * 2 >= len(rows), f"only {len(cmp)} of {len(rows)} index rows equal the oracle's"
    for lnp, out in zip(lnps, outs):
        o_ref, _ = O.sparse_attention_rows(lnp["qa"], oi, cmp, scale=w.scale, d_v=w.d_v, kv=lnp["kv"])
        g = O.bf16_to_f64(host(out))
        assert_attention_close(np.stack([g[b, t] for b, t in cmp]), o_ref)
