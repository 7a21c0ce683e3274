"""lsa_select_streaming_noalloc: the streaming selection with the library's
static device scratch in place of a caller workspace.

It exists for callers that cannot allocate device memory where they select: a
plugin inside a serving engine that has reserved its GPU memory up front for
its own KV cache, or a latency-critical decode path that cannot afford
cudaMalloc/cudaFree (which may block the host and synchronise the device).
Its output must equal the oracle's and lsa_select_streaming's exactly (index
work is compared bit for bit), call after call, although every call reuses the
same scratch.

This file is collected last so that a run stopping at its first failure has
run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import lsa as L
from tests.parity import dev, host


def test_noalloc_rejects_oversized_shape_on_the_host():
    # B*T=21 rows at L_max=1M need just over 16 MiB of selection scratch (20
    # fit); the call must refuse before touching the (fake, never
    # dereferenced) pointers.
    lib = L.load()
    fake = ctypes.c_void_p(256)
    st = lib.lsa_select_streaming_noalloc(fake, fake, 21, 1, 1 << 20, L.Budget(2048, 64, 960), fake, None)
    assert st == L.LSA_ERR_WORKSPACE
    msg = lib.lsa_last_error().decode()
    assert "static scratch" in msg and str(L.LSA_NOALLOC_SCRATCH_BYTES) in msg
    need = L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=21, T=1, L_max=1 << 20)
    assert need > L.LSA_NOALLOC_SCRATCH_BYTES
    fits = L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=20, T=1, L_max=1 << 20)
    assert 0 < fits <= L.LSA_NOALLOC_SCRATCH_BYTES


def test_noalloc_rejects_bad_arguments_on_the_host():
    lib = L.load()
    fake = ctypes.c_void_p(256)
    assert lib.lsa_select_streaming_noalloc(fake, fake, 0, 1, 1024, L.Budget(64, 0, 0), fake, None) \
        == L.LSA_ERR_INVALID_ARG
    assert lib.lsa_select_streaming_noalloc(fake, fake, 1, 1, 1024, L.Budget(64, 40, 40), fake, None) \
        == L.LSA_ERR_INVALID_ARG


def _scores(seed, B, T, L_max, seq_len, ties=False):
    rng = np.random.default_rng(seed)
    if ties:
        sc = (rng.integers(0, 8, size=(B, T, L_max)) * 0.25).astype(np.float32)
    else:
        sc = rng.standard_normal((B, T, L_max)).astype(np.float32)
    for b in range(B):
        for t in range(T):
            sc[b, t, max(0, seq_len[b] - T + t + 1):] = -np.inf   # causal: invisible slots carry -inf
    return sc


# Consecutive calls on the two launch shapes that keep scratch in the static
# buffer. Rows longer than 262144 slots go to the grid-cooperative launch while
# rows x CTAs fit the GPU at once (4 rows of 300000 slots: per-row coordination
# blocks, counters and flags, about 1 MiB); longer rows to the filter launch (15
# rows of 1M slots: the rows' group maxima, candidate pools, per-warp tables and
# counters, about 11.8 MiB, near the limit). Each shape runs twice with new
# scores, interleaved with the other, so the leftovers of one call sit in the
# scratch when the next starts.
SHAPE_A = (4, 1, 300000, (2048, 64, 960))
SHAPE_B = (15, 1, 1 << 20, (2048, 64, 960))
CALLS = [
    (21, SHAPE_A, [300000, 300000, 123457, 299999], True),
    (22, SHAPE_B, [1 << 20] * 12 + [700001, 5000, 1 << 20], False),
    (23, SHAPE_A, [299000, 300000, 300000, 65536], False),
    (24, SHAPE_B, [1 << 20, 999999] + [1 << 20] * 13, True),
]


def test_noalloc_shapes_use_the_static_scratch():
    # guard: if a plan change stopped these shapes from using scratch, the GPU
    # test below would no longer reach the static buffer
    for B, T, L_max, budget in (SHAPE_A, SHAPE_B):
        need = L.workspace_size(L.LSA_OP_SELECT, budget=budget, B=B, T=T, L_max=L_max)
        assert 0 < need <= L.LSA_NOALLOC_SCRATCH_BYTES, (B, L_max, need)


@pytest.mark.gpu
def test_noalloc_select_matches_oracle_and_workspace_select_on_consecutive_calls():
    for seed, (B, T, L_max, budget), seq_len, ties in CALLS:
        sl = np.array(seq_len, np.int32)
        sc = _scores(seed, B, T, L_max, sl, ties)
        sc_d, sl_d = dev(sc, "f32"), dev(sl, "i32")
        idx = torch.full((B, T, budget[0]), -7, dtype=torch.int32, device="cuda")
        L.lsa_select_streaming_noalloc(sc_d, sl_d, budget, idx=idx)
        ref = L.lsa_select_streaming(sc_d, sl_d, budget)
        torch.cuda.synchronize()
        assert L.lsa_device_status() == L.LSA_OK
        got = host(idx)
        assert np.array_equal(got, O.select_streaming(sc, sl, T, *budget)), (seed, B, L_max)
        assert np.array_equal(got, host(ref)), (seed, B, L_max)
