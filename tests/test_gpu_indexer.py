"""Indexer scores (tcgen05 GEMM + fused ReLU/head-weight/causal epilogue) and
flat index sets on the GPU vs the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I
from kv_indexing_b200 import lsa as L
from tests.parity import (accumulation_scale, assert_scores_close, check_index_row, dev, host)

pytestmark = pytest.mark.gpu


def gpu_flat(x, budget, fp8=False):
    if fp8:
        q, k = dev(x["q_idx_fp8"], "e4m3"), dev(x["k_idx_fp8"], "e4m3")
        qs, ks = dev(x["q_scale"], "f32"), dev(x["k_scale"], "f32")
    else:
        q, k = dev(x["q_idx"], "bf16"), dev(x["k_idx"], "bf16")
        qs = ks = None
    w = dev(x["w"], "f32")
    sl = dev(x["seq_len"], "i32")
    B, T = x["q_idx"].shape[:2]
    L_max = x["k_idx"].shape[1]
    scores = torch.empty((B, T, L_max), dtype=torch.float32, device="cuda")
    idx = L.lsa_index_flat(q, w, k, sl, budget, q_scale=qs, k_scale=ks, scores_out=scores)
    torch.cuda.synchronize()
    L.lsa_device_status()
    return host(idx), host(scores)


def check_flat(x, budget, fp8=False):
    gi, gs = gpu_flat(x, budget, fp8)
    kw = dict(fp8=True, q_scale=x["q_scale"], k_scale=x["k_scale"]) if fp8 else {}
    q = x["q_idx_fp8"] if fp8 else x["q_idx"]
    k = x["k_idx_fp8"] if fp8 else x["k_idx"]
    os_ = O.indexer_scores(q, x["w"], k, x["seq_len"], **kw)
    A = accumulation_scale(q, x["w"], k, **kw)
    worst = assert_scores_close(gs, os_, A)
    oi = O.select_streaming(os_, x["seq_len"], q.shape[1], *budget)
    # given identical scores the selection is bit-exact; end to end, near-ties may swap
    B, T = q.shape[:2]
    swaps = 0
    for b in range(B):
        for t in range(T):
            pos = int(x["seq_len"][b]) - T + t
            swaps += check_index_row(gi[b, t], oi[b, t], os_[b, t], pos, budget[1], budget[2])
    return worst, swaps


def small(name, **kw):
    return I.scaled(I.WORKLOADS[name], **kw)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_flat_tiny_workload(seed):
    w = I.WORKLOADS["tiny_l2k"]
    x = I.make_indexer_inputs(w, seed)
    check_flat(x, (w.k, w.sink, w.window))


def test_flat_decode_small_ragged_lengths():
    w = small("flat_decode_128k", B=3, L=8192)
    x = I.make_indexer_inputs(w, 1)
    x["seq_len"] = np.array([8192, 5000, 1900], np.int32)     # ragged: partial last tile, short row
    check_flat(x, (w.k, w.sink, w.window))


def test_flat_prefill_chunk_causal_tiles():
    w = small("prefill_64k", L=4096, T=512, fp8=False)
    x = I.make_indexer_inputs(w, 2)
    check_flat(x, (w.k, w.sink, w.window))


def test_flat_prefill_fp8_keys_and_queries():
    w = small("prefill_64k", L=2048, T=128)
    x = I.make_indexer_inputs(w, 3)
    check_flat(x, (w.k, w.sink, w.window), fp8=True)


@pytest.mark.parametrize("H,d,T", [(8, 64, 3), (16, 128, 5), (32, 64, 1), (128, 128, 2), (4, 128, 1)])
def test_flat_head_and_dim_variants(H, d, T):
    w = I.Workload(name="v", B=2, L=1024, T=T, H=H, d=d, k=128, sink=16, window=16, needles=20)
    x = I.make_indexer_inputs(w, H + d + T)
    check_flat(x, (w.k, w.sink, w.window))
