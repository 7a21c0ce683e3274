"""lsa_select_streaming_noalloc: the streaming selection with the library's
static device scratch in place of a caller workspace.

It exists for callers that cannot allocate device memory where they select: a
plugin inside a serving engine that has reserved its GPU memory up front for
its own KV cache, or a latency-critical decode path that cannot afford
cudaMalloc/cudaFree (which may block the host and synchronise the device).
Its output must equal lsa_select_streaming's exactly (index work is compared
bit for bit), call after call, although every call reuses the same scratch.

This file is collected last so that a run stopping at its first failure has
run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

from kv_indexing_b200 import lsa as L
from tests.parity import dev, host


def test_noalloc_rejects_oversized_shape_on_the_host():
    # B*T=16 rows at L_max=1M need just over 16 MiB of selection scratch; the
    # call must refuse before touching the (fake, never dereferenced) pointers.
    lib = L.load()
    fake = ctypes.c_void_p(256)
    st = lib.lsa_select_streaming_noalloc(fake, fake, 16, 1, 1 << 20, L.Budget(2048, 64, 960), fake, None)
    assert st == L.LSA_ERR_WORKSPACE
    msg = lib.lsa_last_error().decode()
    assert "static scratch" in msg and str(L.LSA_NOALLOC_SCRATCH_BYTES) in msg
    need = L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=16, T=1, L_max=1 << 20)
    assert need > L.LSA_NOALLOC_SCRATCH_BYTES


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


# (seed, B, T, L_max, seq_len, budget, ties): a decode batch at 128K keys, the
# same shape again with new scores (leftover scratch must not leak into it),
# then 160 ragged query rows with heavy ties (more rows than SMs: the other
# launch shape).
CALLS = [
    (11, 8, 1, 131072, [131072, 131072, 100000, 131072, 65536, 131072, 3000, 131072], (2048, 64, 960), False),
    (12, 8, 1, 131072, [131072, 77777, 131072, 131072, 131072, 20000, 131072, 131072], (2048, 64, 960), False),
    (13, 4, 40, 20000, [20000, 9000, 30, 15000], (512, 16, 100), True),
]


@pytest.mark.gpu
def test_noalloc_select_matches_workspace_select_on_consecutive_calls():
    for seed, B, T, L_max, seq_len, budget, ties in CALLS:
        sl = np.array(seq_len, np.int32)
        sc_d = dev(_scores(seed, B, T, L_max, sl, ties), "f32")
        sl_d = dev(sl, "i32")
        idx = torch.full((B, T, budget[0]), -7, dtype=torch.int32, device="cuda")
        L.lsa_select_streaming_noalloc(sc_d, sl_d, budget, idx=idx)
        ref = L.lsa_select_streaming(sc_d, sl_d, budget)
        torch.cuda.synchronize()
        assert L.lsa_device_status() == L.LSA_OK
        assert np.array_equal(host(idx), host(ref)), (seed, B, T, L_max)
