"""Cross-layer group on the GPU: one index set feeds every layer."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I
from kv_indexing_b200 import lsa as L
from tests.parity import assert_attention_close, check_hier_rows, check_index_row, dev, host, same_rows

pytestmark = pytest.mark.gpu


def check_layer_outputs(gi, oi, specs, outs, lses=None):
    """Each layer's GPU output against the oracle's attention over the oracle's
    own index set, on the rows whose GPU index row equals it (the others are
    near-tie swaps judged by the index checks). specs: (inputs, scale, d_v, mla)."""
    rows = same_rows(gi, oi)
    assert len(rows) * 2 >= gi.shape[0] * gi.shape[1], "too few index rows equal the oracle's"
    for i, ((l, scale, d_v, mla), out) in enumerate(zip(specs, outs)):
        kw = dict(kv=l["kv"]) if mla else dict(k=l["k"], v=l["v"])
        o_ref, l_ref = O.sparse_attention_rows(l["qa"], oi, rows, scale=scale, d_v=d_v, **kw)
        g = O.bf16_to_f64(host(out))
        assert_attention_close(np.stack([g[b, t] for b, t in rows]), o_ref)
        if lses is not None:
            gl = host(lses[i])
            assert np.allclose(np.stack([gl[b, t] for b, t in rows]), l_ref, atol=1e-3, rtol=1e-3)


@pytest.mark.parametrize("hier", [False, True])
def test_group_two_layers(hier):
    w = I.scaled(I.WORKLOADS["cli_group_256k"], B=2, L=16384, M=64)
    x = I.make_indexer_inputs(w, 1)
    layers_np = [I.make_attn_inputs(w, 1, layer=i) for i in range(2)]
    q, k, ww = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16"), dev(x["w"], "f32")
    sl = dev(x["seq_len"], "i32")
    budget = (w.k, w.sink, w.window)
    layers = [{"q": dev(l["qa"], "bf16"), "kv": dev(l["kv"], "bf16"), "scale": w.scale, "d_v": w.d_v}
              for l in layers_np]
    P, M = (w.P, w.M) if hier else (0, 0)
    pk = L.lsa_pool_pages(k, sl, w.P) if hier else None
    idx, outs = L.lsa_layer_group(q, ww, k, sl, budget, layers, P=P, M=M, page_keys=pk)
    torch.cuda.synchronize()
    L.lsa_device_status()
    gi = host(idx)
    # the group's index set equals the single indexing call's, bit for bit
    rows = [(b, 0) for b in range(w.B)]
    if hier:
        pages = torch.empty((w.B, 1, M), dtype=torch.int32, device="cuda")
        ref_i, _ = L.lsa_index_hier(q, ww, k, sl, pk, P, M, budget, pages_out=pages)
        torch.cuda.synchronize()
        oi = check_hier_rows(x, x["seq_len"], P, M, budget, gi, host(pages), rows)
    else:
        ref_i = L.lsa_index_flat(q, ww, k, sl, budget)
        torch.cuda.synchronize()
        os_ = O.indexer_scores(x["q_idx"], x["w"], x["k_idx"], x["seq_len"])
        oi = O.select_streaming(os_, x["seq_len"], 1, *budget)
        for b in range(w.B):
            check_index_row(gi[b, 0], oi[b, 0], os_[b, 0], w.L - 1, w.sink, w.window)
    assert np.array_equal(gi, host(ref_i))
    # every layer's output is attention over that set (both layers share one
    # launch, whose split plan differs from a single-layer call's)
    check_layer_outputs(gi, oi, [(lnp, w.scale, w.d_v, True) for lnp in layers_np], outs)


def test_group_mixed_layers_and_launch_chunks():
    """Six layers: MLA runs of equal head count share launches (at most four per
    launch), other layers launch alone. Scales, head counts and lse differ per
    layer, so a layer mixed up inside a shared launch shows in its output."""
    w = I.scaled(I.WORKLOADS["cli_group_256k_flat"], B=2, L=16384)
    x = I.make_indexer_inputs(w, 5)
    sl_np = np.array([16384, 11000], np.int32)
    q, k, ww, sl = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16"), dev(x["w"], "f32"), dev(sl_np, "i32")
    budget = (w.k, w.sink, w.window)
    specs = [I.scaled(w, scale=0.04), I.scaled(w, scale=0.05), I.scaled(w, Hq=64, scale=0.045),
             I.scaled(w, Hq=64, scale=0.035), I.scaled(w, Hq=16, d_qk=64, d_v=64, mla=False, scale=0.125),
             I.scaled(w, scale=0.042)]
    lnps = [I.make_attn_inputs(s, 5, layer=i) for i, s in enumerate(specs)]
    layers = []
    for s_, l in zip(specs, lnps):
        if s_.mla:
            layers.append({"q": dev(l["qa"], "bf16"), "kv": dev(l["kv"], "bf16"), "scale": s_.scale, "d_v": s_.d_v})
        else:
            layers.append({"q": dev(l["qa"], "bf16"), "k": dev(l["k"], "bf16"), "v": dev(l["v"], "bf16"),
                           "scale": s_.scale})
    lses = [torch.empty((w.B, w.T, s_.Hq), dtype=torch.float32, device="cuda") for s_ in specs]
    idx, outs = L.lsa_layer_group(q, ww, k, sl, budget, layers, lses=lses)
    torch.cuda.synchronize()
    L.lsa_device_status()
    gi = host(idx)
    os_ = O.indexer_scores(x["q_idx"], x["w"], x["k_idx"], sl_np)
    oi = O.select_streaming(os_, sl_np, 1, *budget)
    for b in range(w.B):
        check_index_row(gi[b, 0], oi[b, 0], os_[b, 0], int(sl_np[b]) - 1, w.sink, w.window)
    check_layer_outputs(gi, oi, [(l, s_.scale, s_.d_v, s_.mla) for s_, l in zip(specs, lnps)], outs, lses)


def test_group_five_mla_layers():
    """Five MLA layers of one head count: a launch of four, then one of one."""
    w = I.scaled(I.WORKLOADS["cli_group_256k_flat"], B=1, L=8192, T=2)
    x = I.make_indexer_inputs(w, 6)
    q, k, ww, sl = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16"), dev(x["w"], "f32"), dev(x["seq_len"], "i32")
    budget = (w.k, w.sink, w.window)
    scales = [0.03, 0.035, 0.04, 0.045, 0.05]
    lnps = [I.make_attn_inputs(w, 6, layer=i) for i in range(5)]
    layers = [{"q": dev(l["qa"], "bf16"), "kv": dev(l["kv"], "bf16"), "scale": sc, "d_v": w.d_v}
              for l, sc in zip(lnps, scales)]
    idx, outs = L.lsa_layer_group(q, ww, k, sl, budget, layers)
    torch.cuda.synchronize()
    L.lsa_device_status()
    gi = host(idx)
    oi, os_ = O.index_flat(x["q_idx"], x["w"], x["k_idx"], x["seq_len"], budget=w.k, sink=w.sink, window=w.window)
    for t in range(w.T):
        check_index_row(gi[0, t], oi[0, t], os_[0, t], w.L - w.T + t, w.sink, w.window)
    check_layer_outputs(gi, oi, [(l, sc, w.d_v, True) for l, sc in zip(lnps, scales)], outs)


def test_group_rejects_overlapping_outputs():
    w = I.scaled(I.WORKLOADS["cli_group_256k_flat"], B=1, L=4096)
    x = I.make_indexer_inputs(w, 7)
    q, k, ww, sl = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16"), dev(x["w"], "f32"), dev(x["seq_len"], "i32")
    lnps = [I.make_attn_inputs(w, 7, layer=i) for i in range(2)]
    layers = [{"q": dev(l["qa"], "bf16"), "kv": dev(l["kv"], "bf16"), "scale": w.scale, "d_v": w.d_v} for l in lnps]
    big = torch.empty((2 * w.Hq * w.d_v,), dtype=torch.bfloat16, device="cuda")
    shared = big[: w.Hq * w.d_v].view(1, 1, w.Hq, w.d_v)
    shifted = big[w.d_v: w.d_v + w.Hq * w.d_v].view(1, 1, w.Hq, w.d_v)
    with pytest.raises(L.LsaError):
        L.lsa_layer_group(q, ww, k, sl, (w.k, w.sink, w.window), layers, outs=[shared, shifted])
