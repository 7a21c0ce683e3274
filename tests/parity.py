"""Shared helpers for GPU-vs-oracle parity tests (upload, tolerance rules)."""
from __future__ import annotations

import math

import numpy as np

import oracle as O

SCORE_RTOL = 1e-3          # indexer scores: relative to fp32 accumulation
TIE_RTOL = 1e-3            # index sets: swaps allowed within this of the D-th score
ATTN_ATOL = 2e-2           # attention: max-abs
ATTN_RTOL = 1e-2           # attention: ||g - o||_inf / ||o||_inf


def dev(a, kind: str):
    """numpy codes -> torch CUDA tensor of the given kind (bf16 / e4m3 / f32 / i32)."""
    import torch
    if kind == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    if kind == "e4m3":
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e4m3fn).cuda()
    if kind == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    if kind == "i32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    raise ValueError(kind)


def host(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def accumulation_scale(q, w, k, fp8=False, q_scale=None, k_scale=None):
    """A[b,t,s] = sum_h |w| sum_i |q_i k_i| / sqrt(d): the size of the terms the
    fp32 accumulation adds, used to bound the error of scores that cancel."""
    B, T, H, d = q.shape
    if fp8:
        qd = O.e4m3_to_f64(q) * q_scale[..., None]
        kd = O.e4m3_to_f64(k) * k_scale[..., None]
    else:
        qd, kd = O.bf16_to_f64(q), O.bf16_to_f64(k)
    out = np.zeros((B, T, k.shape[1]))
    for b in range(B):
        aq = np.abs(qd[b])                     # [T, H, d]
        ak = np.abs(kd[b])                     # [L, d]
        for t in range(T):
            out[b, t] = (ak @ aq[t].T) @ np.abs(w[b, t]) / math.sqrt(d)
    return out


def assert_scores_close(g, o, A, rows=None):
    """|g - o| <= 1e-3 * max(|o|, 1e-3 * A), and -inf exactly where the oracle has -inf."""
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    neg = np.isneginf(o)
    assert np.array_equal(np.isneginf(g), neg), "masked (-inf) positions differ"
    fin = ~neg
    denom = np.maximum(np.abs(o[fin]), 1e-3 * A[fin])
    err = np.abs(g[fin] - o[fin]) / np.maximum(denom, 1e-30)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= SCORE_RTOL, f"score error {worst:.3g} > {SCORE_RTOL}"
    return worst


def check_index_row(g, o, scores, pos, sink, window, tol=TIE_RTOL):
    """GPU index row g vs oracle row o (both canonical), for a query at ``pos``.

    Validity, checked on g alone: the valid entries come first and the rest is
    -1 padding; no index appears twice; the dynamic block is strictly ascending
    and every entry of it is a dynamic candidate -- inside [sink end, window
    start), so neither sink, window nor beyond pos -- with a finite oracle score
    (``scores`` is -inf at slots that are not candidates). Against the oracle: the
    sink and window lead must match exactly and the valid counts must agree; the
    dynamic blocks may differ only by swaps among candidates whose oracle score
    lies within tol (relative) of the oracle's D-th selected score. Returns the
    number of swapped pairs."""
    g = np.asarray(g)
    o = np.asarray(o)
    assert g.shape == o.shape, f"row lengths differ: {g.shape} vs {o.shape}"
    s_rng, w_rng, c_rng = O.streaming_regions(pos, sink, window)
    n_lead = len(s_rng) + len(w_rng)
    n_valid = int(np.sum(g >= 0))
    assert np.all(g[:n_valid] >= 0) and np.all(g[n_valid:] == -1), "valid entries not followed only by -1 padding"
    gv, ov = g[:n_valid], o[o >= 0]
    assert np.unique(gv).size == gv.size, "an index appears twice"
    assert np.array_equal(g[:n_lead], o[:n_lead]), "sink/window block differs"
    assert gv.size == ov.size, f"valid counts differ: {gv.size} vs {ov.size}"
    gd, od = gv[n_lead:], ov[n_lead:]
    assert np.all(np.diff(gd) > 0), "dynamic block not strictly ascending"
    if gd.size:
        assert gd[0] >= c_rng.start and gd[-1] < c_rng.stop, (
            f"dynamic entries {gd[0]}..{gd[-1]} outside the candidate region [{c_rng.start}, {c_rng.stop})")
        assert np.all(np.asarray(scores, np.float64)[gd] > -np.inf), "a dynamic entry is not a candidate"
    extra = np.setdiff1d(gd, od)
    missing = np.setdiff1d(od, gd)
    if extra.size == 0:
        return 0
    tau = float(np.min(scores[od]))
    band = tol * abs(tau)
    for x in np.concatenate([extra, missing]):
        assert abs(float(scores[x]) - tau) <= band, (
            f"index {x} (score {scores[x]!r}) swapped but not a near-tie of the threshold {tau!r}")
    return int(extra.size)


def assert_attention_close(g, o):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    err = np.abs(g - o)
    mx = float(err.max()) if err.size else 0.0
    rel = mx / max(float(np.abs(o).max()), 1e-30) if err.size else 0.0
    assert mx <= ATTN_ATOL, f"attention max-abs error {mx:.3g}"
    assert rel <= ATTN_RTOL, f"attention relative error {rel:.3g}"
    return mx, rel


def same_rows(gi, oi):
    """(b, t) rows whose GPU index row equals the oracle's bit for bit.

    End-to-end attention parity is checked on those rows, with the oracle
    attending over its own index set: no oracle input ever comes from the GPU.
    (Rows that differ are near-tie swaps, already judged by check_index_row.)"""
    B, T = np.shape(gi)[:2]
    return [(b, t) for b in range(B) for t in range(T) if np.array_equal(gi[b, t], oi[b, t])]


def accumulation_scale_rows(q, w, k, rows, fp8=False, q_scale=None, k_scale=None):
    """accumulation_scale for the listed (b, t) rows only: float64 [len(rows), L]."""
    d = q.shape[3]
    out = []
    for b, t in rows:
        if fp8:
            qd = O.e4m3_to_f64(q[b, t]) * q_scale[b, t][:, None]
            kd = O.e4m3_to_f64(k[b]) * k_scale[b][:, None]
        else:
            qd, kd = O.bf16_to_f64(q[b, t]), O.bf16_to_f64(k[b])
        out.append((np.abs(kd) @ np.abs(qd).T) @ np.abs(w[b, t]) / math.sqrt(d))
    return np.stack(out)


def check_row_valid_over(g, cands, scores, pos, sink, window, tol=TIE_RTOL):
    """A GPU index row g is a valid streaming selection over the candidate set
    ``cands`` (oracle scores ``scores``): the sink and window lead exactly, then
    min(D, |cands|) distinct candidates ascending, then -1 padding; and no
    candidate left out scores above a chosen one by more than tol (relative to
    the lowest chosen score). Used where several selections are correct."""
    g = np.asarray(g)
    s_rng, w_rng, _ = O.streaming_regions(pos, sink, window)
    lead = np.array(list(s_rng) + list(w_rng), dtype=np.int64)
    n = lead.size + min(g.size - lead.size, cands.size)
    assert np.array_equal(g[:lead.size], lead), "sink/window block differs"
    assert np.all(g[lead.size:n] >= 0) and np.all(g[n:] == -1), "wrong count or padding"
    dyn = g[lead.size:n]
    assert np.all(np.diff(dyn) > 0), "dynamic block not strictly ascending"
    assert np.isin(dyn, cands).all(), "a dynamic entry is not a candidate"
    rest = np.setdiff1d(cands, dyn)
    if dyn.size and rest.size:
        tau = float(np.min(scores[dyn]))
        assert float(np.max(scores[rest])) <= tau + tol * abs(tau), "a better candidate was left out"


def check_hier_rows(x, seq_len, P, M, budget, gi, gp, rows, fp8=False):
    """Recalled pages and index rows of the listed (b, t) against the oracle.

    Pages: the forced pages exactly; the others eligible and equal to the
    oracle's up to swaps among pages whose oracle page score lies within 1e-3 of
    the last recalled one. Tokens: the oracle's row (check_index_row) when the
    page sets agree; otherwise a valid selection over the GPU's recalled pages
    by the oracle's token scores (check_row_valid_over). Returns the oracle's
    index rows [B, T, k]."""
    sink, window = budget[1], budget[2]
    T = x["q_idx"].shape[1]
    L_max = x["k_idx"].shape[1]
    kw = dict(P=P, M=M, budget=budget[0], sink=sink, window=window, rows=rows)
    if fp8:   # e4m3 queries, token keys and pooled page keys, each with its scales
        q, k, qs, ks = x["q_idx_fp8"], x["k_idx_fp8"], x["q_scale"], x["k_scale"]
        pk_o, ps_o = O.pool_pages_e4m3(k, ks, seq_len, P)
        oi, op = O.index_hier_e4m3(q, qs, x["w"], k, ks, pk_o, ps_o, seq_len, **kw)
        psc = O.indexer_scores_rows(q, x["w"], pk_o, seq_len, rows, vis_shift=P.bit_length() - 1, L_max=L_max,
                                    fp8=True, q_scale=qs, k_scale=ps_o)
        tsc_all = O.indexer_scores_rows(q, x["w"], k, seq_len, rows, fp8=True, q_scale=qs, k_scale=ks)
    else:
        pk_o = O.pool_pages(x["k_idx"], seq_len, P)
        oi, op = O.index_hier(x["q_idx"], x["w"], x["k_idx"], pk_o, seq_len, **kw)
        psc = O.indexer_scores_rows(x["q_idx"], x["w"], pk_o, seq_len, rows, vis_shift=P.bit_length() - 1,
                                    L_max=L_max)
        tsc_all = O.indexer_scores_rows(x["q_idx"], x["w"], x["k_idx"], seq_len, rows)
    for i, (b, t) in enumerate(rows):
        pos = int(seq_len[b]) - T + t
        if pos < 0:
            assert (gi[b, t] == -1).all() and (gp[b, t] == -1).all()
            continue
        forced, E = O.page_sets(pos, P, sink, window)
        n_g = int(np.sum(gp[b, t] >= 0))
        g_pages, o_pages = gp[b, t][:n_g], op[b, t][op[b, t] >= 0]
        assert np.all(g_pages >= 0) and np.all(gp[b, t][n_g:] == -1), "recalled pages not -1 padded"
        assert np.all(np.diff(g_pages) > 0), "recalled pages not strictly ascending"
        assert g_pages.size == o_pages.size, "recalled page counts differ"
        assert set(forced) <= set(g_pages.tolist()), "a forced page is missing"
        gd, od = np.setdiff1d(g_pages, forced), np.setdiff1d(o_pages, forced)
        assert np.all((gd >= E.start) & (gd < E.stop)), "a recalled page is not eligible"
        _, _, c_rng = O.streaming_regions(pos, sink, window)
        cands = np.arange(c_rng.start, c_rng.stop)
        cands = cands[np.isin(cands // P, g_pages)]
        if np.array_equal(gd, od):
            tsc = np.full(L_max, -np.inf, np.float32)
            tsc[cands] = tsc_all[i][cands]
            check_index_row(gi[b, t], oi[b, t], tsc, pos, sink, window)
        else:
            tau = float(psc[i][od].min())
            for pg in np.setdiff1d(np.union1d(gd, od), np.intersect1d(gd, od)):
                assert abs(float(psc[i][pg]) - tau) <= TIE_RTOL * abs(tau), "page recall differs beyond near-ties"
            check_row_valid_over(gi[b, t], cands, tsc_all[i], pos, sink, window)
    return oi
