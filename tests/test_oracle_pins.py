"""Pins of the CPU oracle to things other than itself (no GPU).

Each test ties one oracle function to a value the pages or mathematics fix: a
hand-worked example (tests/golden), a closed form on a constructed input, a
library routine (torch's bf16 / e4m3 conversions, scaled_dot_product_attention),
brute force on tiny inputs, or an invariant the method implies.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from kv_indexing_b200 import inputs as I

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def bf16(x):
    """Exact small values -> bf16 codes (test helper; values used are exact)."""
    return I.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


# ---------------------------------------------------------------------------
# element codecs
# ---------------------------------------------------------------------------


def test_bf16_rne_known_patterns():
    cases = {
        0x3F800000: 0x3F80,   # 1.0
        0x3F808000: 0x3F80,   # 1 + 2^-8: tie, upper even -> down
        0x3F818000: 0x3F82,   # 1 + 3*2^-8: tie, upper odd -> up
        0x3F808001: 0x3F81,   # just above the tie -> up
        0x3F807FFF: 0x3F80,   # just below the tie -> down
        0xC0200000: 0xC020,   # -2.5
        0x7F7FFFFF: 0x7F80,   # FLT_MAX rounds to +inf
        0x7F800000: 0x7F80,   # +inf
        0x80000000: 0x8000,   # -0
    }
    u = np.array(list(cases.keys()), dtype=np.uint32)
    got = O.f32_to_bf16_rne(u.view(np.float32))
    assert [int(g) for g in got] == list(cases.values())
    nan = O.f32_to_bf16_rne(np.array([np.nan], np.float32))
    assert (int(nan[0]) & 0x7F80) == 0x7F80 and (int(nan[0]) & 0x7F) != 0


def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        rng.standard_normal(1000).astype(np.float32) * 1e-30])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.f32_to_bf16_rne(x), ref)
    assert np.array_equal(I.f32_to_bf16_bits(x), ref)       # the input generator too
    back = O.bf16_to_f64(ref)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_e4m3_decode_known_codes():
    vals = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
            0x38: 1.0, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0, 0x3C: 1.5}
    got = O.e4m3_to_f64(np.array(list(vals.keys()), np.uint8))
    assert got.tolist() == list(vals.values())
    assert np.isnan(O.e4m3_to_f64(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = O.e4m3_to_f64(codes)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_input_e4m3_encoder_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(50000) * 100, rng.standard_normal(5000) * 0.01,
                        [448.0, -448.0, 0.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10]]).astype(np.float32)
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(I.f32_to_e4m3_bits(x), ref)


@pytest.mark.parametrize("shape", [(5,), (3, 7, 64), (2, 4001, 16)])
def test_input_e4m3_row_quantiser_is_per_row_amax_over_448(shape):
    # scale = amax / 448 per row (1 for an all-zero row), codes = torch's e4m3 of
    # x / scale; rows are encoded in chunks, which must not change a byte
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(shape) * 5).astype(np.float32)
    x.reshape(-1, shape[-1])[0] = 0
    t = torch.from_numpy(x)
    amax = t.abs().amax(dim=-1)
    sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    ref = (t / sc[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for chunk in (1 << 14, 997):
        codes, scale = I.quantize_e4m3_rows(x, chunk_rows=chunk)
        assert codes.shape == x.shape and scale.shape == x.shape[:-1]
        assert np.array_equal(scale, sc.numpy()) and np.array_equal(codes, ref)


# ---------------------------------------------------------------------------
# indexer score
# ---------------------------------------------------------------------------


def test_score_closed_form_single_head():
    q = O.bf16_to_f64(bf16([[1.0, 0.0]]))
    k = O.bf16_to_f64(bf16([[3.0, 4.0], [-3.0, 4.0]]))
    s = O.indexer_scores_row(q, np.array([0.5]), k, 2)
    assert s[0] == np.float32(0.5 * 3 / math.sqrt(2))
    assert s[1] == 0.0                      # negative dot -> ReLU -> exactly 0


def test_score_handworked_golden():
    g = json.load(open(os.path.join(GOLD, "handworked_flat.json")))
    q = np.array(g["q"], np.float64)
    k = np.array(g["keys"], np.float64)
    s = O.indexer_scores_row(q, np.array(g["w"]), k, 8)
    assert s.tolist() == g["scores_pos7"]
    s5 = O.indexer_scores_row(q, np.array(g["w"]), k, 6)
    assert s5[:6].tolist() == g["scores_pos7"][:6] and np.isneginf(s5[6:]).all()


def test_score_basis_keys_pick_columns():
    # keys = unit vectors e_i  =>  dot[i, h] = q[h, i]: score_i = sum_h w_h relu(q[h,i]) / sqrt(d).
    # A transposed operand or a wrong reduction axis breaks this.
    rng = np.random.default_rng(1)
    H, d = 5, 8
    q = O.bf16_to_f64(I.normal_bf16((H, d), rng))
    w = rng.random(H)
    s = O.indexer_scores_row(q, w, np.eye(d), d)
    for i in range(d):
        expect = sum(w[h] * max(q[h, i], 0.0) for h in range(H)) / math.sqrt(d)
        assert s[i] == np.float32(expect)


def test_score_brute_force_tiny():
    rng = np.random.default_rng(2)
    H, d, n = 3, 4, 6
    qb = I.normal_bf16((H, d), rng)
    kb = I.normal_bf16((n, d), rng)
    w = rng.random(H).astype(np.float32)
    q, k = O.bf16_to_f64(qb), O.bf16_to_f64(kb)
    s = O.indexer_scores_row(q, w.astype(np.float64), k, n)
    for si in range(n):
        tot = 0.0
        for h in range(H):
            dot = 0.0
            for i in range(d):
                dot += q[h][i] * k[si][i]
            tot += float(w[h]) * (dot if dot > 0 else 0.0)
        assert abs(float(s[si]) - tot / math.sqrt(d)) <= 1e-6 * abs(tot) + 1e-30


def test_score_head_permutation_and_homogeneity():
    rng = np.random.default_rng(4)
    H, d, n = 8, 16, 50
    q = O.bf16_to_f64(I.normal_bf16((H, d), rng))
    k = O.bf16_to_f64(I.normal_bf16((n, d), rng))
    w = rng.random(H)
    base = O.indexer_scores_row(q, w, k, n)
    perm = rng.permutation(H)
    assert np.allclose(O.indexer_scores_row(q[perm], w[perm], k, n), base, rtol=1e-6)
    # scaling head 3 by 2 adds exactly that head's term once more
    q2 = q.copy(); q2[3] *= 2.0
    only3 = O.indexer_scores_row(q[3:4], w[3:4], k, n)
    assert np.allclose(O.indexer_scores_row(q2, w, k, n), base.astype(np.float64) + only3, rtol=1e-6)


def test_score_fp8_scale_identity():
    rng = np.random.default_rng(5)
    B, T, H, d, L = 1, 2, 4, 16, 40
    q8 = I.f32_to_e4m3_bits(rng.standard_normal((B, T, H, d)) * 3)
    k8 = I.f32_to_e4m3_bits(rng.standard_normal((B, L, d)) * 3)
    w = rng.random((B, T, H)).astype(np.float32)
    ks = (rng.random((B, L)) + 0.5).astype(np.float32)
    qs = (rng.random((B, T, H)) + 0.5).astype(np.float32)
    sl = np.array([L], np.int32)
    with_scale = O.indexer_scores(q8, w, k8, sl, q_scale=qs, k_scale=ks, fp8=True)
    no_kscale = O.indexer_scores(q8, w, k8, sl, q_scale=qs, k_scale=np.ones_like(ks), fp8=True)
    vis = np.isfinite(with_scale)
    assert np.allclose(with_scale[vis], (no_kscale * ks[:, None, :])[vis], rtol=1e-6)
    # per-(t,h) query scale acts like a weight on that head
    folded = O.indexer_scores(q8, w * qs, k8, sl, q_scale=np.ones_like(qs), k_scale=ks, fp8=True)
    assert np.allclose(with_scale[vis], folded[vis], rtol=1e-6)


def test_score_causal_mask():
    rng = np.random.default_rng(6)
    B, T, H, d, L = 2, 5, 2, 8, 30
    q = I.normal_bf16((B, T, H, d), rng)
    k = I.normal_bf16((B, L + 4, d), rng)
    w = rng.random((B, T, H)).astype(np.float32)
    sl = np.array([L, L - 7], np.int32)
    sc = O.indexer_scores(q, w, k, sl)
    for b in range(B):
        for t in range(T):
            pos = sl[b] - T + t
            assert np.isfinite(sc[b, t, :pos + 1]).all()
            assert np.isneginf(sc[b, t, pos + 1:]).all()


# ---------------------------------------------------------------------------
# streaming selection
# ---------------------------------------------------------------------------


def test_select_handworked_golden():
    g = json.load(open(os.path.join(GOLD, "handworked_flat.json")))
    q = np.array(g["q"], np.float64)
    k = np.array(g["keys"], np.float64)
    for c in g["cases"]:
        sc = O.indexer_scores_row(q, np.array(g["w"]), k, c["pos"] + 1)
        got = O.select_streaming_row(sc, c["pos"], c["k"], c["sink"], c["window"])
        assert got.tolist() == c["idx"], c


def _brute_select(scores, pos, k, S, W):
    """Rank counting: candidate i is chosen iff fewer than D candidates beat it,
    where j beats i when s_j > s_i or (s_j == s_i and j < i)."""
    sink = [s for s in range(0, min(S, pos + 1))]
    win = [s for s in range(max(0, pos - W + 1), pos + 1) if s not in sink]
    cand = [s for s in range(0, pos + 1) if s not in sink and s not in win]
    D = k - len(sink) - len(win)
    chosen = []
    for i in cand:
        beats = 0
        for j in cand:
            if scores[j] > scores[i] or (scores[j] == scores[i] and j < i):
                beats += 1
        if beats < D:
            chosen.append(i)
    out = sink + win + sorted(chosen)
    return out + [-1] * (k - len(out))


@pytest.mark.parametrize("seed", range(6))
def test_select_brute_force_with_ties(seed):
    rng = np.random.default_rng(100 + seed)
    n = 40
    for pos, k, S, W in itertools.product([0, 3, 9, 25, 39], [4, 8, 16], [0, 2, 4], [0, 1, 3]):
        if S + W > k:
            continue
        sc = (rng.integers(0, 4, size=n) * 0.5).astype(np.float32)   # heavy ties
        sc[rng.integers(0, n)] = -0.0
        got = O.select_streaming_row(sc, pos, k, S, W)
        assert got.tolist() == _brute_select(sc.tolist(), pos, k, S, W), (pos, k, S, W)


def test_select_closed_forms():
    n, pos, k, S, W = 1000, 999, 64, 8, 24
    C = list(range(S, pos - W + 1))
    D = k - S - W
    inc = np.arange(n, dtype=np.float32)                     # score = index
    got = O.select_streaming_row(inc, pos, k, S, W)
    assert got[S + W:].tolist() == C[-D:]                    # largest indices win
    dec = -np.arange(n, dtype=np.float32)
    got = O.select_streaming_row(dec, pos, k, S, W)
    assert got[S + W:].tolist() == C[:D]
    flat = np.full(n, 2.0, np.float32)                       # all tied: lowest indices
    got = O.select_streaming_row(flat, pos, k, S, W)
    assert got[S + W:].tolist() == C[:D]


def test_select_invariants_random():
    rng = np.random.default_rng(9)
    for _ in range(200):
        n = int(rng.integers(1, 300))
        pos = int(rng.integers(-1, n))
        k = int(rng.integers(1, 64))
        S = int(rng.integers(0, k + 1))
        W = int(rng.integers(0, k - S + 1))
        sc = rng.standard_normal(n).astype(np.float32)
        got = O.select_streaming_row(sc, pos, k, S, W)
        valid = got[got >= 0]
        assert valid.size == min(k, pos + 1)
        assert len(set(valid.tolist())) == valid.size
        assert (valid <= pos).all()
        assert (got[valid.size:] == -1).all()
        s_rng, w_rng, _ = O.streaming_regions(pos, S, W)
        lead = list(s_rng) + list(w_rng)
        assert got[:len(lead)].tolist() == lead          # sink then window, always present
        dyn = got[len(lead):valid.size]
        assert (np.diff(dyn) > 0).all()


# ---------------------------------------------------------------------------
# page pooling
# ---------------------------------------------------------------------------


def test_pool_closed_forms():
    P, d = 16, 8
    L = 3 * P + 5                                   # 3 full pages + a partial one
    kb = np.zeros((1, L, d), np.uint16)
    kb[0, :P] = bf16(np.full((P, d), 1.25))         # constant page -> same constant
    rows = np.arange(P, dtype=np.float32)[:, None] * np.float32(2 ** -6)
    kb[0, P:2 * P] = bf16(np.broadcast_to(rows, (P, d)))          # mean = (P-1)/2 * 2^-6
    kb[0, 2 * P:3 * P] = bf16(np.full((P, d), -3.0))
    kb[0, 3 * P:] = bf16(np.full((5, d), 7.0))
    pk = O.pool_pages(kb, np.array([L], np.int32), P)
    assert pk.shape == (1, L // P, d)
    assert (O.bf16_to_f64(pk[0, 0]) == 1.25).all()
    assert (O.bf16_to_f64(pk[0, 1]) == (P - 1) / 2 * 2 ** -6).all()
    assert (O.bf16_to_f64(pk[0, 2]) == -3.0).all()


def test_pool_rounds_to_nearest_even():
    # two rows: the exact mean sits on a bf16 tie; RNE picks the even neighbour
    kb = bf16([[[1.0], [1.0 + 2 ** -7], [1.0 + 2 ** -7], [1.0 + 2 * 2 ** -7]]])
    pk = O.pool_pages(kb, np.array([4], np.int32), 2)
    assert pk[0, 0, 0] == 0x3F80          # 1 + 2^-8 -> even 1.0
    assert pk[0, 1, 0] == 0x3F82          # 1 + 3*2^-8 -> even 1 + 2^-6


def test_pool_float32_sequential_sum():
    # float32 order matters: 2^24 + 1 + 1 - 2^24 is 0 left to right in float32
    big = float(2 ** 24)
    kb = bf16([[[big], [1.0], [1.0], [-big]]])
    pk = O.pool_pages(kb, np.array([4], np.int32), 4)
    assert O.bf16_to_f64(pk[0, 0])[0] == 0.0


# ---------------------------------------------------------------------------
# hierarchical indexing
# ---------------------------------------------------------------------------


def test_hier_handworked_golden():
    gf = json.load(open(os.path.join(GOLD, "handworked_flat.json")))
    gh = json.load(open(os.path.join(GOLD, "handworked_hier.json")))
    q = np.array(gf["q"], np.float64)
    k = np.array(gf["keys"], np.float64)
    kb = bf16(np.array(gf["keys"], np.float32))[None]
    pk = O.pool_pages(kb, np.array([8], np.int32), gh["P"])
    assert np.array_equal(O.bf16_to_f64(pk[0]), np.array(gh["page_keys"]))
    ps = O.indexer_scores_row(q, np.array(gf["w"]), O.bf16_to_f64(pk[0]), 4)
    assert ps.tolist() == gh["page_scores"]
    for c in gh["cases"]:
        idx, pages = O.index_hier_row(q, np.array(gf["w"]), k, O.bf16_to_f64(pk[0]), c["pos"],
                                      gh["P"], c["M"], c["k"], c["sink"], c["window"])
        assert idx.tolist() == c["idx"]
        assert pages[pages >= 0].tolist() == c["pages"]


def _rand_case(rng, B=1, T=3, H=4, d=16, L=500):
    q = I.normal_bf16((B, T, H, d), rng)
    k = I.normal_bf16((B, L, d), rng)
    w = rng.random((B, T, H)).astype(np.float32)
    return q, w, k, np.array([L] * B, np.int32)


@pytest.mark.parametrize("P,L", [(4, 128), (8, 203), (16, 512)])
def test_hier_full_recall_equals_flat(P, L):
    rng = np.random.default_rng(P + L)
    q, w, k, sl = _rand_case(rng, T=4, L=L)
    kk, S, W = 64, 8, 24
    pk = O.pool_pages(k, sl, P)
    M = -(-L // P) + 2                       # M*P >= L: every page recalled
    idx_f, _ = O.index_flat(q, w, k, sl, budget=kk, sink=S, window=W)
    idx_h, pages = O.index_hier(q, w, k, pk, sl, P=P, M=M, budget=kk, sink=S, window=W)
    assert np.array_equal(idx_f, idx_h)


def test_hier_page_size_one_equals_flat():
    rng = np.random.default_rng(11)
    q, w, k, sl = _rand_case(rng, T=3, L=300)
    kk, S, W = 48, 4, 12
    pk = O.pool_pages(k, sl, 1)
    assert np.array_equal(pk, k)                 # mean of one bf16 row is that row
    D = kk - S - W
    M = D + S + W                                # M >= D + |F|
    idx_f, _ = O.index_flat(q, w, k, sl, budget=kk, sink=S, window=W)
    idx_h, _ = O.index_hier(q, w, k, pk, sl, P=1, M=M, budget=kk, sink=S, window=W)
    assert np.array_equal(idx_f, idx_h)


def test_hier_recalls_planted_page_and_forced_pages():
    rng = np.random.default_rng(12)
    P, L, d, H = 16, 1024, 32, 4
    q, w, k, sl = _rand_case(rng, T=1, H=H, d=d, L=L)
    target = 20                                   # a page well inside the dynamic region
    qf = O.bf16_to_f64(q[0, 0, 1])
    k[0, target * P:(target + 1) * P] = bf16(np.broadcast_to(qf, (P, d)))
    pk = O.pool_pages(k, sl, P)
    S, W, kk, M = 16, 48, 128, 8
    idx, pages = O.index_hier(q, w, k, pk, sl, P=P, M=M, budget=kk, sink=S, window=W)
    pg = pages[0, 0][pages[0, 0] >= 0].tolist()
    forced, _ = O.page_sets(L - 1, P, S, W)
    assert target in pg
    assert set(forced) <= set(pg) and len(pg) == M and pg == sorted(pg)


def test_hier_forced_page_count_1m_geometry():
    # 1M context, P=64, sink 64, window 960: 1 sink page + 15 window pages
    pos = 1048575
    forced, E = O.page_sets(pos, 64, 64, 960)
    assert len(forced) == 16 and forced[0] == 0 and forced[1] == (pos - 959) // 64
    assert E.start == 1 and E.stop == (pos - 959) // 64


# ---------------------------------------------------------------------------
# sparse attention
# ---------------------------------------------------------------------------


def test_attention_handworked_golden():
    g = json.load(open(os.path.join(GOLD, "handworked_attention.json")))
    for c in g["cases"]:
        o, lse = O.sparse_attention_row(np.array(c["q"], float), np.array(c["K"], float),
                                        np.array(c["V"], float), np.array(c["idx"]), c["scale"])
        assert np.allclose(o, np.array(c["o"]), rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, np.array(c["lse"]), rtol=1e-12, atol=1e-12)


def test_attention_select_all_equals_dense_sdpa():
    rng = np.random.default_rng(21)
    B, T, Hq, dqk, dv, L = 1, 6, 4, 32, 16, 40
    qa = I.normal_bf16((B, T, Hq, dqk), rng)
    kk = I.normal_bf16((B, L, dqk), rng)
    vv = I.normal_bf16((B, L, dv), rng)
    sl = np.array([L], np.int32)
    scale = 0.17
    idx = np.full((B, T, L), -1, np.int32)
    for t in range(T):
        pos = L - T + t
        idx[0, t, :pos + 1] = rng.permutation(pos + 1)        # all visible, any order
    o, lse = O.sparse_attention(qa, idx, sl, scale=scale, d_v=dv, k=kk, v=vv)
    qt = torch.from_numpy(O.bf16_to_f64(qa[0])).permute(1, 0, 2)         # [Hq, T, dqk]
    kt = torch.from_numpy(O.bf16_to_f64(kk[0]))[None].expand(Hq, L, dqk)
    vt = torch.from_numpy(O.bf16_to_f64(vv[0]))[None].expand(Hq, L, dv)
    mask = torch.zeros(T, L, dtype=torch.bool)
    for t in range(T):
        mask[t, :L - T + t + 1] = True
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    assert np.allclose(o[0], ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_attention_single_index_and_identical_keys_and_permutation():
    rng = np.random.default_rng(22)
    Hq, dqk, dv, L = 3, 8, 8, 20
    qa = O.bf16_to_f64(I.normal_bf16((Hq, dqk), rng))
    K = O.bf16_to_f64(I.normal_bf16((L, dqk), rng))
    V = O.bf16_to_f64(I.normal_bf16((L, dv), rng))
    o, lse = O.sparse_attention_row(qa, K, V, np.array([7, -1, -1, -1]), 0.5)
    assert np.array_equal(o, np.broadcast_to(V[7], (Hq, dv)))
    assert np.allclose(lse, 0.5 * qa @ K[7])
    Ksame = np.broadcast_to(K[0], (L, dqk)).copy()
    sel = np.array([1, 4, 9, 11])
    o, lse = O.sparse_attention_row(qa, Ksame, V, sel, 0.5)
    assert np.allclose(o, np.broadcast_to(V[sel].mean(0), (Hq, dv)), rtol=1e-12)
    assert np.allclose(lse, 0.5 * qa @ K[0] + math.log(4))
    idx = rng.permutation(L)[:10]
    o1, l1 = O.sparse_attention_row(qa, K, V, idx, 0.3)
    o2, l2 = O.sparse_attention_row(qa, K, V, idx[::-1].copy(), 0.3)
    assert np.allclose(o1, o2, rtol=1e-12) and np.allclose(l1, l2, rtol=1e-12)
    o, lse = O.sparse_attention_row(qa, K, V, np.array([-1, -1]), 0.3)
    assert (o == 0).all() and np.isneginf(lse).all()


def test_attention_mla_alias_v_is_prefix_of_latent_row():
    rng = np.random.default_rng(23)
    B, T, Hq, dqk, dv, L = 1, 2, 2, 24, 16, 30
    qa = I.normal_bf16((B, T, Hq, dqk), rng)
    kv = I.normal_bf16((B, L, dqk), rng)
    sl = np.array([L], np.int32)
    idx = np.stack([rng.permutation(L - 2)[:8], rng.permutation(L - 1)[:8]])[None].astype(np.int32)
    o1, l1 = O.sparse_attention(qa, idx, sl, scale=0.2, d_v=dv, kv=kv)
    o2, l2 = O.sparse_attention(qa, idx, sl, scale=0.2, d_v=dv, k=kv, v=kv[..., :dv].copy())
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_attention_e4m3_kv_equals_dense_sdpa_on_dequantised_rows():
    # e4m3 latent cache: K = code * scale (torch's e4m3 decode, float64), V its
    # first d_v columns; selecting every visible row must equal dense SDPA
    rng = np.random.default_rng(24)
    B, T, Hq, dqk, dv, L = 1, 5, 3, 32, 16, 36
    qa = I.normal_bf16((B, T, Hq, dqk), rng)
    kv8, ks = I.quantize_e4m3_rows(rng.standard_normal((B, L, dqk)).astype(np.float32) * 3)
    idx = np.full((B, T, L), -1, np.int32)
    for t in range(T):
        pos = L - T + t
        idx[0, t, :pos + 1] = rng.permutation(pos + 1)
    o, lse = O.sparse_attention_e4m3_rows(qa, idx, None, scale=0.21, d_v=dv, kv8=kv8, k_scale=ks)
    kdq = torch.from_numpy(kv8[0].copy()).view(torch.float8_e4m3fn).to(torch.float64) * \
        torch.from_numpy(ks[0].astype(np.float64))[:, None]
    qt = torch.from_numpy(O.bf16_to_f64(qa[0])).permute(1, 0, 2)
    mask = torch.zeros(T, L, dtype=torch.bool)
    for t in range(T):
        mask[t, :L - T + t + 1] = True
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kdq[None].expand(Hq, L, dqk),
                                                           kdq[None, :, :dv].expand(Hq, L, dv), attn_mask=mask,
                                                           scale=0.21)
    assert np.allclose(o.reshape(T, Hq, dv), ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_attention_e4m3_kv_single_index_returns_the_scaled_row():
    rng = np.random.default_rng(25)
    Hq, dqk, dv, L = 2, 16, 8, 10
    qa = I.normal_bf16((1, 1, Hq, dqk), rng)
    kv8 = rng.integers(0, 256, (1, L, dqk)).astype(np.uint8)
    kv8[(kv8 & 0x7F) == 0x7F] = 0x01                                # no NaN codes
    ks = np.full((1, L), 0.375, np.float32)
    o, lse = O.sparse_attention_e4m3_rows(qa, np.array([[[4, -1, -1]]], np.int32), None, scale=0.5, d_v=dv,
                                          kv8=kv8, k_scale=ks)
    row = O.e4m3_to_f64(kv8[0, 4]) * 0.375
    assert np.array_equal(o[0], np.broadcast_to(row[:dv], (Hq, dv)))
    assert np.allclose(lse[0], 0.5 * O.bf16_to_f64(qa[0, 0]) @ row, rtol=1e-13)


# ---------------------------------------------------------------------------
# cross-layer group
# ---------------------------------------------------------------------------


def test_layer_group_shares_index_and_matches_single_layers():
    rng = np.random.default_rng(31)
    q, w, k, sl = _rand_case(rng, T=2, L=200)
    layers = []
    for li in range(2):
        layers.append({"qa": I.normal_bf16((1, 2, 4, 16), rng), "kv": I.normal_bf16((1, 200, 16), rng),
                       "scale": 0.25, "d_v": 8})
    idx, outs = O.layer_group(q, w, k, sl, layers, budget=40, sink=4, window=8)
    idx1, _ = O.index_flat(q, w, k, sl, budget=40, sink=4, window=8)
    assert np.array_equal(idx, idx1)
    for lay, (o, lse) in zip(layers, outs):
        o1, l1 = O.sparse_attention(lay["qa"], idx1, sl, scale=0.25, d_v=8, kv=lay["kv"])
        assert np.array_equal(o, o1) and np.array_equal(lse, l1)


def test_input_needles_are_planted_in_dynamic_region():
    w = I.scaled(I.WORKLOADS["tiny_l2k"])
    x = I.make_indexer_inputs(w, seed=1)
    npos = x["needle_pos"][0]
    npos = npos[npos >= 0]
    assert npos.size == w.n_needles
    assert (npos >= w.sink).all() and (npos <= w.L - 1 - w.window).all()


# ---------------------------------------------------------------------------
# compressed-entry indexing
# ---------------------------------------------------------------------------


def test_compressed_entry_one_token_equals_flat():
    rng = np.random.default_rng(21)
    B, T, H, d, L = 2, 3, 4, 16, 96
    q = I.normal_bf16((B, T, H, d), rng)
    k = I.normal_bf16((B, L, d), rng)
    w = rng.random((B, T, H)).astype(np.float32)
    sl = np.array([L, 70], np.int32)
    gi, gs = O.index_compressed(q, w, k, sl, m=1, budget=24, sink=4, window=6)
    fi, fs = O.index_flat(q, w, k, sl, budget=24, sink=4, window=6)
    assert np.array_equal(gi, fi)
    assert np.array_equal(gs, fs)


def test_compressed_entry_visibility_by_membership():
    """An entry is scored iff every token it stands for is visible."""
    rng = np.random.default_rng(22)
    B, T, H, d, m, n_e = 1, 9, 2, 8, 4, 12
    q = I.normal_bf16((B, T, H, d), rng)
    ek = I.normal_bf16((B, n_e, d), rng)
    w = rng.random((B, T, H)).astype(np.float32)
    sl = np.array([37], np.int32)                    # queries at tokens 28 .. 36
    _, sc = O.index_compressed(q, w, ek, sl, m=m, budget=8, sink=1, window=2)
    for t in range(T):
        pos = 37 - T + t
        for e in range(n_e):
            complete = all(tok <= pos for tok in range(e * m, e * m + m))
            assert np.isfinite(sc[0, t, e]) == complete, (pos, e)


def test_compressed_entry_closed_form():
    """Entry keys (e, 0), q = (1, 0), w = 1: score = e / sqrt(2), so the
    dynamic block takes the highest complete entries. m = 4, token 41: entries
    0..9 are complete; sink {0, 1}, window {7, 8, 9}, D = 2 -> {5, 6}."""
    n_e, m = 12, 4
    ek = np.zeros((1, n_e, 2), np.float32)
    ek[0, :, 0] = np.arange(n_e)
    q = np.array([[[[1.0, 0.0]]]], np.float32)
    w = np.ones((1, 1, 1), np.float32)
    idx, sc = O.index_compressed(bf16(q), w, bf16(ek), np.array([42], np.int32), m=m, budget=7, sink=2,
                                 window=3)
    assert idx[0, 0].tolist() == [0, 1, 7, 8, 9, 5, 6]
    assert np.allclose(sc[0, 0, :10], np.arange(10) / math.sqrt(2.0), rtol=1e-6)
    assert np.isneginf(sc[0, 0, 10:]).all()


@pytest.mark.parametrize("seed", range(3))
def test_compressed_entry_select_brute_force(seed):
    rng = np.random.default_rng(300 + seed)
    B, T, H, d, m, n_e = 1, 6, 1, 4, 8, 40
    q = bf16(np.ones((B, T, H, d)))
    ek = bf16(rng.integers(0, 3, size=(B, n_e, d)).astype(np.float32) * 0.5)   # many tied scores
    w = np.ones((B, T, H), np.float32)
    sl = np.array([n_e * m - 5], np.int32)
    idx, sc = O.index_compressed(q, w, ek, sl, m=m, budget=12, sink=2, window=3)
    for t in range(T):
        pe = (int(sl[0]) - T + t + 1) // m - 1
        assert idx[0, t].tolist() == _brute_select(sc[0, t].tolist(), pe, 12, 2, 3)


def test_compressed_inputs_plant_needles_in_dynamic_entries():
    """Entry needles sit in the decode query's dynamic entries (between the sink
    entries and the window entries of its last complete entry), and every index
    the oracle picks there is a complete, visible entry."""
    w = I.scaled(I.WORKLOADS["compressed_decode_1m"], B=1, L=32768, needle_frac=0.0, needles=12)
    x = I.make_compressed_inputs(w, seed=2)
    n_e = w.L // w.m
    assert x["entry_keys"].shape == (1, n_e, w.d) and int(x["seq_len"][0]) == w.L
    npos = x["needle_pos"][0]
    npos = npos[npos >= 0]
    pe = O.entry_position(w.L - 1, w.m)
    assert npos.size == 12 and (npos >= w.sink).all() and (npos <= pe - w.window).all()
    idx, _ = O.index_compressed(x["q_idx"], x["w"], x["entry_keys"], x["seq_len"], m=w.m, budget=w.k,
                                sink=w.sink, window=w.window)
    sel = idx[0, 0][idx[0, 0] >= 0]
    assert sel.size == w.k and (sel <= pe).all() and np.unique(sel).size == sel.size


# ---------------------------------------------------------------------------
# FP8 hierarchical indexing (oracle only; no kernel path yet)
# ---------------------------------------------------------------------------


def test_oracle_e4m3_encoder_matches_torch():
    rng = np.random.default_rng(31)
    x = np.concatenate([rng.standard_normal(40000) * 50, rng.standard_normal(4000) * 0.01,
                        [0.0, -0.0, 448.0, -448.0, 2.0 ** -9, 3 * 2.0 ** -10, 5 * 2.0 ** -10, 17.0, 19.0, 240.0]])
    x = np.clip(x, -448.0, 448.0).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.f64_to_e4m3_rne(x), ref)
    assert O.f64_to_e4m3_rne(np.array([500.0, -1e6]))[0] == 0x7E           # saturating
    assert O.f64_to_e4m3_rne(np.array([-1e6]))[0] == 0xFE


def test_pool_pages_e4m3_closed_form():
    # one full page of P = 4 identical tokens [1, 2, 0.5, -1] (scale 1): the mean is
    # the same row, amax 2 -> page scale 2/448, codes of 224, 448, 112, -224
    row = O.f64_to_e4m3_rne(np.array([1.0, 2.0, 0.5, -1.0]))
    k8 = np.tile(row, (1, 6, 1)).astype(np.uint8)                              # 6 tokens: page 1 is partial
    ks = np.ones((1, 6), np.float32)
    codes, scales = O.pool_pages_e4m3(k8, ks, np.array([6], np.int32), 4)
    assert codes.shape == (1, 1, 4) and scales[0, 0] == np.float32(2.0) / np.float32(448.0)
    assert O.e4m3_to_f64(codes[0, 0]).tolist() == [224.0, 448.0, 112.0, -224.0]
    # token scales act before the mean: halving every token's scale halves the page scale only
    codes2, scales2 = O.pool_pages_e4m3(k8, ks * np.float32(0.5), np.array([6], np.int32), 4)
    assert np.array_equal(codes2, codes) and scales2[0, 0] == scales[0, 0] * np.float32(0.5)
    # a page whose tokens differ: the mean of the dequantized rows, then quantized
    k8b = O.f64_to_e4m3_rne(np.array([[[1.0, 0.0]], [[3.0, 0.0]], [[2.0, 4.0]], [[2.0, 0.0]]]).reshape(1, 4, 2))
    cb, sb = O.pool_pages_e4m3(k8b, np.ones((1, 4), np.float32), np.array([4], np.int32), 4)
    assert sb[0, 0] == np.float32(2.0) / np.float32(448.0)                     # mean row (2, 1): amax 2
    assert O.e4m3_to_f64(cb[0, 0]).tolist() == [448.0, 224.0]


@pytest.mark.parametrize("P,L", [(4, 128), (16, 512)])
def test_hier_e4m3_full_recall_equals_flat_e4m3(P, L):
    rng = np.random.default_rng(7 * P + L)
    B, T, H, d = 2, 3, 4, 32
    q8, qs = I.quantize_e4m3_rows(rng.standard_normal((B, T, H, d)).astype(np.float32))
    k8, ks = I.quantize_e4m3_rows(rng.standard_normal((B, L, d)).astype(np.float32))
    w = rng.random((B, T, H)).astype(np.float32)
    sl = np.array([L, L - 9], np.int32)
    kk, S, W = 48, 4, 12
    pc, ps = O.pool_pages_e4m3(k8, ks, sl, P)
    M = -(-L // P) + 2                                                         # M * P >= L: every page recalled
    idx_f, _ = O.index_flat(q8, w, k8, sl, budget=kk, sink=S, window=W, q_scale=qs, k_scale=ks, fp8=True)
    idx_h, pages = O.index_hier_e4m3(q8, qs, w, k8, ks, pc, ps, sl, P=P, M=M, budget=kk, sink=S, window=W)
    assert np.array_equal(idx_f, idx_h)


def test_hier_e4m3_recalls_a_planted_page():
    """A page whose P tokens all copy one query head's vector scores highest among
    the eligible pages for that query, so a recall of one dynamic page takes it."""
    rng = np.random.default_rng(41)
    B, T, H, d, L, P = 1, 1, 2, 32, 512, 16
    qf = rng.standard_normal((B, T, H, d)).astype(np.float32)
    kf = rng.standard_normal((B, L, d)).astype(np.float32) * 0.3
    kf[0, 10 * P:11 * P] = qf[0, 0, 0] * 2.0                                     # page 10
    q8, qs = I.quantize_e4m3_rows(qf)
    k8, ks = I.quantize_e4m3_rows(kf)
    w = np.array([[[1.0, 0.0]]], np.float32)                                    # only head 0 counts
    sl = np.array([L], np.int32)
    pc, ps = O.pool_pages_e4m3(k8, ks, sl, P)
    S, W = 16, 16                                                               # forced pages: 0 and 31
    idx, pages = O.index_hier_e4m3(q8, qs, w, k8, ks, pc, ps, sl, P=P, M=3, budget=64, sink=S, window=W)
    assert pages[0, 0].tolist() == [0, 10, 31]
    assert set(range(10 * P, 11 * P)) <= set(idx[0, 0].tolist())
