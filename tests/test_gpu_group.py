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
    # and every layer's output equals a separate sparse-attention call on that set
    for lay, lnp, out in zip(layers, layers_np, outs):
        o1, _ = L.lsa_sparse_attn(lay["q"], idx, sl, w.scale, kv=lay["kv"], d_v=w.d_v)
        torch.cuda.synchronize()
        assert torch.equal(o1, out)
        o_ref, _ = O.sparse_attention(lnp["qa"], gi, x["seq_len"], scale=w.scale, d_v=w.d_v, kv=lnp["kv"])
        assert_attention_close(O.bf16_to_f64(host(out)), o_ref)
    if not hier:
        os_ = O.indexer_scores(x["q_idx"], x["w"], x["k_idx"], x["seq_len"])
        oi = O.select_streaming(os_, x["seq_len"], 1, *budget)
        for b in range(w.B):
            check_index_row(gi[b, 0], oi[b, 0], os_[b, 0], lead_count(w.L - 1, w.sink, w.window))
