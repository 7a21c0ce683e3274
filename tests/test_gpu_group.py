"""Cross-layer group on the GPU: one index set feeds every layer."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I
from kv_indexing_b200 import lsa as L
from tests.parity import assert_attention_close, check_index_row, dev, host, lead_count

pytestmark = pytest.mark.gpu


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
    if hier:
        ref_i, _ = L.lsa_index_hier(q, ww, k, sl, pk, P, M, budget)
    else:
        ref_i = L.lsa_index_flat(q, ww, k, sl, budget)
    torch.cuda.synchronize()
    assert np.array_equal(gi, host(ref_i))
    # and every layer's output is attention over that set (both layers share one
    # launch, whose split plan differs from a single-layer call's)
    for lnp, out in zip(layers_np, outs):
        o_ref, _ = O.sparse_attention(lnp["qa"], gi, x["seq_len"], scale=w.scale, d_v=w.d_v, kv=lnp["kv"])
        assert_attention_close(O.bf16_to_f64(host(out)), o_ref)
    if not hier:
        os_ = O.indexer_scores(x["q_idx"], x["w"], x["k_idx"], x["seq_len"])
        oi = O.select_streaming(os_, x["seq_len"], 1, *budget)
        for b in range(w.B):
            check_index_row(gi[b, 0], oi[b, 0], os_[b, 0], lead_count(w.L - 1, w.sink, w.window))


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
        check_index_row(gi[b, 0], oi[b, 0], os_[b, 0], lead_count(int(sl_np[b]) - 1, w.sink, w.window))
    for s_, l, out, lse in zip(specs, lnps, outs, lses):
        if s_.mla:
            o_ref, l_ref = O.sparse_attention(l["qa"], gi, sl_np, scale=s_.scale, d_v=s_.d_v, kv=l["kv"])
        else:
            o_ref, l_ref = O.sparse_attention(l["qa"], gi, sl_np, scale=s_.scale, d_v=s_.d_v, k=l["k"], v=l["v"])
        assert_attention_close(O.bf16_to_f64(host(out)), o_ref)
        assert np.allclose(host(lse), l_ref, atol=1e-3, rtol=1e-3)


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
    for l, sc, out in zip(lnps, scales, outs):
        o_ref, _ = O.sparse_attention(l["qa"], gi, x["seq_len"], scale=sc, d_v=w.d_v, kv=l["kv"])
        assert_attention_close(O.bf16_to_f64(host(out)), o_ref)


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
