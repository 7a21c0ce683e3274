"""Sparse MQA / MLA attention on the GPU vs the oracle (2e-2 max-abs, 1e-2 relative)."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I
from kv_indexing_b200 import lsa as L
from tests.parity import assert_attention_close, dev, host

pytestmark = pytest.mark.gpu


def rand_idx(rng, B, T, k, L, seq_len, n_valid=None):
    idx = np.full((B, T, k), -1, np.int32)
    for b in range(B):
        for t in range(T):
            pos = int(seq_len[b]) - T + t
            nv = min(k, pos + 1) if n_valid is None else min(n_valid, pos + 1)
            if nv > 0:
                idx[b, t, :nv] = np.sort(rng.choice(pos + 1, size=nv, replace=False))
    return idx


def run(w, x, idx, seq_len):
    sl = dev(seq_len, "i32")
    q = dev(x["qa"], "bf16")
    lse = torch.empty(idx.shape[:2] + (w.Hq,), dtype=torch.float32, device="cuda")
    if w.mla:
        out, _ = L.lsa_sparse_attn(q, dev(idx, "i32"), sl, w.scale, kv=dev(x["kv"], "bf16"), d_v=w.d_v, lse=lse)
    else:
        out, _ = L.lsa_sparse_attn(q, dev(idx, "i32"), sl, w.scale, k=dev(x["k"], "bf16"), v=dev(x["v"], "bf16"),
                                   lse=lse)
    torch.cuda.synchronize()
    L.lsa_device_status()
    return O.bf16_to_f64(host(out)), host(lse)


def oracle_attn(w, x, idx, seq_len):
    if w.mla:
        return O.sparse_attention(x["qa"], idx, seq_len, scale=w.scale, d_v=w.d_v, kv=x["kv"])
    return O.sparse_attention(x["qa"], idx, seq_len, scale=w.scale, d_v=w.d_v, k=x["k"], v=x["v"])


@pytest.mark.parametrize("seed", [1, 2])
def test_attention_tiny_mqa(seed):
    w = I.WORKLOADS["tiny_l2k"]
    rng = np.random.default_rng(seed)
    x = I.make_attn_inputs(w, seed)
    sl = np.array([w.L], np.int32)
    idx = rand_idx(rng, w.B, w.T, w.k, w.L, sl)
    g, gl = run(w, x, idx, sl)
    o, ol = oracle_attn(w, x, idx, sl)
    assert_attention_close(g, o)
    assert np.allclose(gl, ol, atol=1e-3, rtol=1e-3)


def test_attention_mla_decode_splits():
    w = I.scaled(I.WORKLOADS["flat_decode_128k"], B=2, L=8192)
    rng = np.random.default_rng(3)
    x = I.make_attn_inputs(w, 3)
    sl = np.array([8192, 6000], np.int32)
    idx = rand_idx(rng, w.B, w.T, w.k, w.L, sl)
    g, gl = run(w, x, idx, sl)
    o, ol = oracle_attn(w, x, idx, sl)
    assert_attention_close(g, o)
    assert np.allclose(gl, ol, atol=1e-3, rtol=1e-3)


def test_attention_mla_many_rows_padding_and_empty():
    w = I.scaled(I.WORKLOADS["flat_decode_128k"], B=1, L=4096, T=40)
    rng = np.random.default_rng(4)
    x = I.make_attn_inputs(w, 4)
    sl = np.array([4096], np.int32)
    idx = rand_idx(rng, w.B, w.T, w.k, w.L, sl, n_valid=700)    # -1 padded tails
    idx[0, 5] = -1                                               # a row with nothing selected
    g, gl = run(w, x, idx, sl)
    o, ol = oracle_attn(w, x, idx, sl)
    assert_attention_close(g, o)
    assert (g[0, 5] == 0).all() and np.isneginf(gl[0, 5]).all()
    fin = np.isfinite(ol)
    assert np.allclose(gl[fin], ol[fin], atol=1e-3, rtol=1e-3)


def test_attention_select_all_equals_dense():
    # k >= pos + 1 with every visible token selected == dense causal attention
    w = I.Workload(name="dense", B=1, L=256, T=8, H=4, d=64, k=256, sink=0, window=0, Hq=16, d_qk=64, d_v=64,
                   mla=False, scale=0.125)
    x = I.make_attn_inputs(w, 9)
    sl = np.array([256], np.int32)
    idx = np.full((1, 8, 256), -1, np.int32)
    for t in range(8):
        idx[0, t, :256 - 8 + t + 1] = np.arange(256 - 8 + t + 1)
    g, _ = run(w, x, idx, sl)
    qt = torch.from_numpy(O.bf16_to_f64(x["qa"][0])).permute(1, 0, 2)
    kt = torch.from_numpy(O.bf16_to_f64(x["k"][0]))[None].expand(16, 256, 64)
    vt = torch.from_numpy(O.bf16_to_f64(x["v"][0]))[None].expand(16, 256, 64)
    mask = torch.zeros(8, 256, dtype=torch.bool)
    for t in range(8):
        mask[t, :256 - 8 + t + 1] = True
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.125)
    assert_attention_close(g[0], ref.permute(1, 0, 2).numpy())


def test_attention_streaming_prefix_promise_matches_reading_idx():
    # Index rows from the streaming selection; the attention computes their sink
    # and window prefix itself when promised (and splits the row differently), so
    # both paths must match the oracle within the attention tolerance.
    w = I.scaled(I.WORKLOADS["flat_decode_128k"], B=3, L=8192)
    x = I.make_attn_inputs(w, 11)
    sl = np.array([8192, 5000, 900], np.int32)
    rng = np.random.default_rng(12)
    sc = rng.standard_normal((3, 1, 8192)).astype(np.float32)
    for b in range(3):
        sc[b, 0, sl[b]:] = -np.inf
    budget = (w.k, w.sink, w.window)
    sl_d, q, kv = dev(sl, "i32"), dev(x["qa"], "bf16"), dev(x["kv"], "bf16")
    oi = O.select_streaming(sc, sl, 1, *budget)          # the rows the selection writes for these scores
    assert np.array_equal(host(L.lsa_select_streaming(dev(sc, "f32"), sl_d, budget)), oi)
    idx = dev(oi, "i32")
    lse1 = torch.empty((3, 1, w.Hq), dtype=torch.float32, device="cuda")
    lse2 = torch.empty_like(lse1)
    o1, _ = L.lsa_sparse_attn(q, idx, sl_d, w.scale, kv=kv, d_v=w.d_v, lse=lse1)
    o2, _ = L.lsa_sparse_attn(q, idx, sl_d, w.scale, kv=kv, d_v=w.d_v, lse=lse2, stream_budget=budget)
    torch.cuda.synchronize()
    L.lsa_device_status()
    o, ol = oracle_attn(w, x, oi, sl)
    assert_attention_close(O.bf16_to_f64(host(o1)), o)
    assert_attention_close(O.bf16_to_f64(host(o2)), o)
    assert np.allclose(host(lse2), ol, atol=1e-3, rtol=1e-3)
    assert np.allclose(host(lse1), host(lse2), atol=1e-3, rtol=1e-3)


@pytest.mark.parametrize("mla", [True, False])
def test_attention_out_of_range_index_is_skipped_and_flagged(mla):
    # entries >= L_max are skipped by the kernel and flagged in the device status
    # word: lsa_device_status reports LSA_ERR_INVALID_ARG once, then clears
    if mla:
        w = I.scaled(I.WORKLOADS["flat_decode_128k"], B=1, L=4096, T=2)
    else:
        w = I.scaled(I.WORKLOADS["tiny_l2k"], T=2)
    x = I.make_attn_inputs(w, 21)
    sl = np.array([w.L], np.int32)
    rng = np.random.default_rng(21)
    idx = rand_idx(rng, w.B, w.T, w.k, w.L, sl, n_valid=min(w.k, 300))
    bad = idx.copy()
    bad[0, 0, 5] = w.L            # first slot past the cache
    bad[0, 1, 17] = w.L + 999
    sl_d = dev(sl, "i32")
    q = dev(x["qa"], "bf16")
    L.lsa_device_status()         # start clean
    if mla:
        out, _ = L.lsa_sparse_attn(q, dev(bad, "i32"), sl_d, w.scale, kv=dev(x["kv"], "bf16"), d_v=w.d_v)
    else:
        out, _ = L.lsa_sparse_attn(q, dev(bad, "i32"), sl_d, w.scale, k=dev(x["k"], "bf16"), v=dev(x["v"], "bf16"))
    torch.cuda.synchronize()
    with pytest.raises(L.LsaError) as e:
        L.lsa_device_status()
    assert e.value.status == L.LSA_ERR_INVALID_ARG
    assert L.lsa_device_status() == L.LSA_OK        # cleared by the read
    skipped = bad.copy()
    skipped[skipped >= w.L] = -1                    # what the kernel computes: the row without those entries
    o_ref, _ = oracle_attn(w, x, skipped, sl)
    assert_attention_close(O.bf16_to_f64(host(out)), o_ref)


# ---- FP8 latent cache (e4m3 codes with a per-token scale): K = V = code * scale

def kv_e4m3(x):
    """The workload's latent rows quantised per token (scale = amax / 448)."""
    return I.quantize_e4m3_rows(I.bf16_bits_to_f32(x["kv"]))


def run_e4m3(w, x, kv8, ks, idx, seq_len, stream_budget=None):
    sl = dev(seq_len, "i32")
    lse = torch.empty(idx.shape[:2] + (w.Hq,), dtype=torch.float32, device="cuda")
    out, _ = L.lsa_sparse_attn(dev(x["qa"], "bf16"), dev(idx, "i32"), sl, w.scale, kv=dev(kv8, "e4m3"),
                               kv_scale=dev(ks, "f32"), d_v=w.d_v, lse=lse, stream_budget=stream_budget)
    torch.cuda.synchronize()
    L.lsa_device_status()
    return O.bf16_to_f64(host(out)), host(lse)


@pytest.mark.parametrize("B,L_,T,n_valid", [(2, 8192, 1, None), (1, 4096, 40, 700), (2, 2048, 3, 5)])
def test_attention_mla_e4m3_kv_matches_oracle(B, L_, T, n_valid):
    # splits, ragged lengths, -1 padding and an empty row, against the oracle's
    # attention over the dequantised cache
    w = I.scaled(I.WORKLOADS["flat_decode_128k"], B=B, L=L_, T=T)
    rng = np.random.default_rng(31 + B + T)
    x = I.make_attn_inputs(w, 31)
    kv8, ks = kv_e4m3(x)
    sl = np.array([L_, L_ - 1234][:B], np.int32)
    idx = rand_idx(rng, w.B, w.T, w.k, w.L, sl, n_valid=n_valid)
    if T > 2:
        idx[0, 1] = -1
    g, gl = run_e4m3(w, x, kv8, ks, idx, sl)
    o, ol = O.sparse_attention_e4m3_rows(x["qa"], idx, None, scale=w.scale, d_v=w.d_v, kv8=kv8, k_scale=ks)
    o, ol = o.reshape(g.shape), ol.reshape(gl.shape)
    assert_attention_close(g, o)
    fin = np.isfinite(ol)
    assert np.allclose(gl[fin], ol[fin], atol=1e-3, rtol=1e-3)
    if T > 2:
        assert (g[0, 1] == 0).all() and np.isneginf(gl[0, 1]).all()


def test_attention_mla_e4m3_kv_streaming_prefix_and_bad_index():
    w = I.scaled(I.WORKLOADS["flat_decode_128k"], B=2, L=8192)
    x = I.make_attn_inputs(w, 33)
    kv8, ks = kv_e4m3(x)
    sl = np.array([8192, 3000], np.int32)
    rng = np.random.default_rng(33)
    sc = rng.standard_normal((2, 1, 8192)).astype(np.float32)
    for b in range(2):
        sc[b, 0, sl[b]:] = -np.inf
    budget = (w.k, w.sink, w.window)
    oi = O.select_streaming(sc, sl, 1, *budget)
    g, _ = run_e4m3(w, x, kv8, ks, oi, sl, stream_budget=budget)      # prefix computed, not read
    o, _ = O.sparse_attention_e4m3_rows(x["qa"], oi, None, scale=w.scale, d_v=w.d_v, kv8=kv8, k_scale=ks)
    assert_attention_close(g, o.reshape(g.shape))
    bad = oi.copy()
    bad[1, 0, 1500] = w.L + 7
    L.lsa_device_status()
    L.lsa_sparse_attn(dev(x["qa"], "bf16"), dev(bad, "i32"), dev(sl, "i32"), w.scale, kv=dev(kv8, "e4m3"),
                      kv_scale=dev(ks, "f32"), d_v=w.d_v)
    torch.cuda.synchronize()
    with pytest.raises(L.LsaError) as e:
        L.lsa_device_status()
    assert e.value.status == L.LSA_ERR_INVALID_ARG


def test_layer_group_e4m3_kv_layers():
    # two layers with their own e4m3 caches share one attention launch
    w = I.scaled(I.WORKLOADS["cli_group_256k"], B=2, L=8192)
    xi = I.make_indexer_inputs(w, 35)
    lnps = [I.make_attn_inputs(w, 35, layer=i) for i in range(2)]
    quant = [kv_e4m3(l) for l in lnps]
    budget = (w.k, w.sink, w.window)
    q, k, ww, sl = dev(xi["q_idx"], "bf16"), dev(xi["k_idx"], "bf16"), dev(xi["w"], "f32"), dev(xi["seq_len"], "i32")
    layers = [{"q": dev(l["qa"], "bf16"), "kv": dev(kv8, "e4m3"), "kv_scale": dev(ks, "f32"), "scale": w.scale,
               "d_v": w.d_v} for l, (kv8, ks) in zip(lnps, quant)]
    idx, outs = L.lsa_layer_group(q, ww, k, sl, budget, layers)
    torch.cuda.synchronize()
    L.lsa_device_status()
    gi = host(idx)
    for l, (kv8, ks), out in zip(lnps, quant, outs):
        o, _ = O.sparse_attention_e4m3_rows(l["qa"], gi, None, scale=w.scale, d_v=w.d_v, kv8=kv8, k_scale=ks)
        g = O.bf16_to_f64(host(out))
        assert_attention_close(g, o.reshape(g.shape))
