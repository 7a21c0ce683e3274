"""A second restatement of the LSA oracle in numpy/BLAS, kept as a cross-check.

The oracle of record is the plain C++ in ``oracle/lsa_oracle.cpp`` (loaded by
``oracle/__init__.py``). This module computes the same definitions
independently, through numpy and BLAS, and ``tests/test_oracle_cross_check.py``
holds the two to each other function by function.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module. The
product path (the C-ABI library and its Python binding) never calls it, and it
shares no code, table or helper with the CUDA sources.

Everything here is the plain definition written out with numpy, in float64
unless a step fixes another precision, slow and meant to be read against the
pages:

* "LongCat Sparse Attention: Taming the Lightning via Streaming-aware
  Hierarchical Cross-Layer Indexing" (arXiv 2608.01662; summary page) --
  abstract (SI, CLI, HI), key contributions (HI: O(L) -> O(L/P + MP) per query),
  limitations (SI gives 50% of the budget to fixed regions).
* "LongCat-Flash-Lite-Sparse" model card -- the SI / CLI / HI bullets.
* "DSA Lightning Indexer" article (Baidu AI Cloud) -- "Lightweight Scoring
  Module", "Dynamic Token Selector", "Sparse Attention Calculator".

Readings taken where the pages are silent (each restated where it is used):

R1  Indexer score with head weights: score[t,s] = sum_h w[t,h]*ReLU(q[t,h].k[s])/sqrt(d).
    The article's scoring module shows the single-head ReLU(QK^T/sqrt(d)); the LSA
    paper's section 2.2 recaps the DSA mechanism, whose indexer sums heads with
    per-query weights w. ReLU(x)/sqrt(d) == ReLU(x/sqrt(d)), so the placement of
    the scale does not matter.
R2  Causality: key s is visible to the query at absolute position pos iff s <= pos.
    The T queries of a sequence of length L sit at pos = L-T .. L-1.
R3  Streaming regions: sink = [0, min(S, pos+1)); window = the W most recent
    visible tokens, minus any already in the sink; dynamic candidates = visible
    tokens in neither. D = k - |sink| - |window| dynamic slots.
R4  Top-k order: score descending, ties to the lower index (the article's
    torch.topk leaves ties unspecified).
R5  Output layout: sink ascending, window ascending, dynamic ascending, then -1
    padding up to k (fewer visible tokens than k => everything visible is taken).
R6  Page pooling: page p = tokens [pP, pP+P); only full pages are pooled; the
    mean is a float32 sum in ascending row order, one float32 division by P,
    then bf16 round-to-nearest-even. The pooled key is a stored bf16 code, so
    the oracle takes that decision in the precision the kernel stores it in.
R7  Hierarchical recall: forced pages F = pages that hold sink or window tokens;
    eligible pages E = full, fully visible pages holding only dynamic
    candidates; recall R = F + the top (M - |F|) of E by page score (ties to the
    lower page). Fine candidates = dynamic candidates inside R; then R3-R5.
R8  Sparse attention: o[h] = sum_j softmax_j(scale * qa[h].K[idx_j]) V[idx_j]
    over the valid (non -1) indices; lse = natural log of the softmax
    denominator plus the max. No valid index: o = 0, lse = -inf. For MLA, V is
    the first d_v columns of the latent row.
R9  Cross-layer indexing: one index set per query, computed once from the
    group's indexer inputs, feeds every layer of the group.
R10 FP8 keys/queries: the value of an e4m3 code times its float32 row scale.
R11 Compressed entries (the DSA article's "Technical Evolution": the indexer
    picks top-k entries of compressed historical representations): entry e
    stands for tokens [e m, e m + m) and exists once all m are cached, so the
    query at pos sees entries e < (pos + 1) // m. Its key is given (the pages
    name no compressor). Scores are R1 on the entry keys; the selection is
    R3-R5 over entries, at entry position (pos + 1) // m - 1, with budget, sink
    and window counted in entries. m = 1 is flat indexing.
R12 FP8 hierarchical indexing (the pages only name "quantized computation"):
    token keys and queries as R10. A page key is the float32 mean of its
    tokens' dequantized keys (R6's order and division), stored as e4m3 with a
    float32 page scale amax / 448 (round to nearest even, saturating), like
    the token keys. Page and fine scores are R1 on the dequantized values;
    recall and selection as R7.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

NEG_INF32 = np.float32(-np.inf)


# ---------------------------------------------------------------------------
# Element decoding / encoding
# ---------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64. A bf16 is the upper half of a float32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern: keep the top 16 bits, round the dropped 16 bits
    to nearest with ties to even (a carry may reach the exponent; that is the
    correct rounding up to the next binade or to infinity). NaN stays a quiet NaN."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    upper = u >> np.uint64(16)
    lower = u & np.uint64(0xFFFF)
    half = np.uint64(0x8000)
    up = (lower > half) | ((lower == half) & ((upper & np.uint64(1)) == np.uint64(1)))
    r = upper + up.astype(np.uint64)
    is_nan = (u & np.uint64(0x7FFFFFFF)) > np.uint64(0x7F800000)
    r = np.where(is_nan, upper | np.uint64(0x0040), r)
    return r.astype(np.uint16)


def _e4m3_table():
    """The 127 non-negative finite e4m3 values, ascending, and their codes."""
    codes = np.arange(0x7F, dtype=np.uint8)
    return e4m3_to_f64(codes), codes


def f64_to_e4m3_rne(x: np.ndarray) -> np.ndarray:
    """Real value -> e4m3 code: the nearest finite e4m3 value, ties to the even
    code, magnitudes beyond 448 saturating to 448; the sign bit follows x (-0
    included). Written as a search over the value table, not bit arithmetic."""
    vals, codes = _e4m3_table()
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), vals[-1])
    hi = np.clip(np.searchsorted(vals, a, side="left"), 0, vals.size - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - vals[lo], vals[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((codes[hi] & 1) == 0))
    c = np.where(pick_hi, codes[hi], codes[lo]).astype(np.uint8)
    c = np.where(a == vals[hi], codes[hi], c).astype(np.uint8)
    return (c | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)).astype(np.uint8)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3 code -> float64.

    Layout s.eeee.mmm, exponent bias 7. Exponent field 0: subnormal m/8 * 2^-6.
    Otherwise (1 + m/8) * 2^(e-7). Codes with all seven low bits set are NaN.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    sub = m / 8.0 * 2.0 ** -6
    nor = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    v = np.where(e == 0, sub, nor)
    v = np.where((c & 0x7F) == 0x7F, np.nan, v)
    return sign * v


# ---------------------------------------------------------------------------
# Lightning-indexer score (article: "Lightweight Scoring Module"; R1, R2, R10)
# ---------------------------------------------------------------------------


def indexer_scores_row(q_row: np.ndarray, w_row: np.ndarray, keys: np.ndarray,
                       n_visible: int) -> np.ndarray:
    """Scores of one query against ``keys`` (float64 [n, d]).

    q_row: float64 [H, d]; w_row: float64 [H]. Keys 0 .. n_visible-1 are visible
    (R2); the rest get -inf. Returns float32 [n].

        dot[s, h]  = sum_i keys[s, i] * q_row[h, i]        (float64)
        score[s]   = sum_h w_row[h] * max(dot[s, h], 0) / sqrt(d)
    """
    n, d = keys.shape
    out = np.full((n,), NEG_INF32, dtype=np.float32)
    nv = max(0, min(int(n_visible), n))
    if nv == 0:
        return out
    dots = keys[:nv] @ q_row.T                       # [nv, H]
    relu = np.maximum(dots, 0.0)
    score = (relu @ w_row) / math.sqrt(d)
    out[:nv] = score.astype(np.float32)
    return out


def _decode_q(q, q_scale, fp8: bool) -> np.ndarray:
    if fp8:
        return e4m3_to_f64(q) * np.asarray(q_scale, np.float64)[..., None]
    return bf16_to_f64(q)


def _decode_k(k, k_scale, fp8: bool) -> np.ndarray:
    if fp8:
        return e4m3_to_f64(k) * np.asarray(k_scale, np.float64)[..., None]
    return bf16_to_f64(k)


def indexer_scores(q: np.ndarray, w: np.ndarray, k: np.ndarray, seq_len: np.ndarray,
                   *, q_scale=None, k_scale=None, fp8: bool = False,
                   rows: Optional[list] = None) -> np.ndarray:
    """Flat indexer scores for a batch.

    q [B,T,H,d], w [B,T,H], k [B,L_max,d] (bf16 codes, or e4m3 codes with
    q_scale [B,T,H] / k_scale [B,L_max]). Returns float32 [B,T,L_max] with -inf at
    invisible slots. ``rows`` optionally restricts work to a list of (b, t); the
    other rows are left at -inf.
    """
    B, T, H, d = q.shape
    L_max = k.shape[1]
    out = np.full((B, T, L_max), NEG_INF32, dtype=np.float32)
    todo = rows if rows is not None else [(b, t) for b in range(B) for t in range(T)]
    by_b = {}
    for b, t in todo:
        by_b.setdefault(b, []).append(t)
    for b, ts in by_b.items():
        L = int(min(max(int(seq_len[b]), 0), L_max))
        kd = _decode_k(k[b, :L], None if k_scale is None else k_scale[b, :L], fp8)
        for t in ts:
            pos = L - T + t
            if pos < 0:
                continue
            qd = _decode_q(q[b, t], None if q_scale is None else q_scale[b, t], fp8)
            out[b, t, :L] = indexer_scores_row(qd, np.asarray(w[b, t], np.float64), kd, pos + 1)
    return out


# ---------------------------------------------------------------------------
# Streaming-aware selection (LSA abstract (1), model card "SI"; article
# "Dynamic Token Selector"; R3, R4, R5)
# ---------------------------------------------------------------------------


def streaming_regions(pos: int, sink: int, window: int) -> Tuple[range, range, range]:
    """(sink, window, dynamic-candidate) token ranges for a query at ``pos`` (R3)."""
    if pos < 0:
        return range(0), range(0), range(0)
    sink_end = min(sink, pos + 1)
    w_lo = max(sink_end, pos - window + 1)
    return range(0, sink_end), range(w_lo, pos + 1), range(sink_end, w_lo)


def top_by_score(cands: np.ndarray, scores: np.ndarray, n: int) -> np.ndarray:
    """The first ``n`` of ``cands`` ordered by (score descending, index ascending)
    (R4), returned in ascending index order (R5)."""
    cands = np.asarray(cands, dtype=np.int64)
    if n <= 0 or cands.size == 0:
        return np.zeros((0,), dtype=np.int64)
    s = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((cands, -s))      # primary key: -score; secondary: index
    return np.sort(cands[order[:n]])


def select_streaming_row(scores: np.ndarray, pos: int, k: int, sink: int,
                         window: int) -> np.ndarray:
    """Index set of one query from its float32 score row (R3-R5).

    Dynamic candidates with a score of -inf are not candidates (only invisible
    slots carry -inf)."""
    out = np.full((k,), -1, dtype=np.int32)
    s_rng, w_rng, c_rng = streaming_regions(pos, sink, window)
    fixed = list(s_rng) + list(w_rng)
    D = k - len(fixed)
    if D < 0:
        raise ValueError("sink + window exceed the budget")
    cands = np.arange(c_rng.start, c_rng.stop, dtype=np.int64)
    sc = scores[cands] if cands.size else np.zeros((0,), np.float32)
    keep = sc > NEG_INF32
    dyn = top_by_score(cands[keep], sc[keep], D)
    sel = np.concatenate([np.asarray(fixed, dtype=np.int64), dyn])
    out[:sel.size] = sel
    return out


def select_streaming(scores: np.ndarray, seq_len: np.ndarray, T: int, k: int,
                     sink: int, window: int) -> np.ndarray:
    """Batch form: scores [B,T,L_max] float32 -> idx [B,T,k] int32."""
    B = scores.shape[0]
    L_max = scores.shape[2]
    out = np.full((B, T, k), -1, dtype=np.int32)
    for b in range(B):
        L = int(min(max(int(seq_len[b]), 0), L_max))
        for t in range(T):
            out[b, t] = select_streaming_row(scores[b, t], L - T + t, k, sink, window)
    return out


def index_flat(q, w, k, seq_len, *, budget: int, sink: int, window: int,
               q_scale=None, k_scale=None, fp8: bool = False):
    """Flat indexing: scores, then streaming selection. Returns (idx, scores)."""
    sc = indexer_scores(q, w, k, seq_len, q_scale=q_scale, k_scale=k_scale, fp8=fp8)
    idx = select_streaming(sc, seq_len, q.shape[1], budget, sink, window)
    return idx, sc


# ---------------------------------------------------------------------------
# Hierarchical indexing (LSA abstract (3); key contributions: coarse-to-fine,
# O(L/P + MP) per query; model card "HI"; R6, R7)
# ---------------------------------------------------------------------------


def pool_pages(k_bits: np.ndarray, seq_len: np.ndarray, P: int) -> np.ndarray:
    """Mean-pooled page keys (R6).

    k_bits [B, L_max, d] bf16 codes -> [B, L_max // P, d] bf16 codes. Pages that
    are not full (p*P + P > L) are not pooled and are returned as 0.
    """
    B, L_max, d = k_bits.shape
    n_pages = L_max // P
    out = np.zeros((B, n_pages, d), dtype=np.uint16)
    for b in range(B):
        L = int(min(max(int(seq_len[b]), 0), L_max))
        n_full = L // P
        if n_full == 0:
            continue
        x = (k_bits[b, :n_full * P].astype(np.uint32) << np.uint32(16)).view(np.float32)
        x = x.reshape(n_full, P, d)
        acc = np.zeros((n_full, d), dtype=np.float32)
        for j in range(P):                      # float32 adds, ascending row order
            acc = (acc + x[:, j, :]).astype(np.float32)
        mean = (acc / np.float32(P)).astype(np.float32)
        out[b, :n_full] = f32_to_bf16_rne(mean)
    return out


def page_sets(pos: int, P: int, sink: int, window: int):
    """Forced pages F (sorted list) and the eligible page range E for ``pos`` (R7)."""
    s_rng, w_rng, _ = streaming_regions(pos, sink, window)
    sink_end = s_rng.stop
    e_lo = -(-sink_end // P)                      # ceil(|sink| / P)
    forced = set(range(0, e_lo))
    if len(w_rng) > 0:
        forced |= set(range(w_rng.start // P, pos // P + 1))
        e_hi = w_rng.start // P
    else:
        e_hi = (pos + 1) // P
    return sorted(forced), range(e_lo, max(e_lo, e_hi))


def index_hier_row(q_row: np.ndarray, w_row: np.ndarray, keys: np.ndarray,
                   page_keys: np.ndarray, pos: int, P: int, M: int, k: int,
                   sink: int, window: int):
    """Coarse-to-fine selection of one query (R7). Returns (idx [k], pages [M]).

    keys: float64 [L, d] (this sequence); page_keys: float64 [n_pages, d].
    pages: the recalled pages in ascending order, -1 padded to M.
    """
    idx = np.full((k,), -1, dtype=np.int32)
    pages_out = np.full((M,), -1, dtype=np.int32)
    if pos < 0:
        return idx, pages_out
    forced, E = page_sets(pos, P, sink, window)
    n_dyn = M - len(forced)
    if n_dyn < 0:
        raise ValueError("recall M smaller than the forced sink/window pages")
    e_pages = np.arange(E.start, E.stop, dtype=np.int64)
    if e_pages.size:
        psc = indexer_scores_row(q_row, w_row, page_keys[E.start:E.stop], E.stop - E.start)
        chosen = top_by_score(e_pages, psc, n_dyn)
    else:
        chosen = np.zeros((0,), np.int64)
    recall = np.sort(np.concatenate([np.asarray(forced, np.int64), chosen]))
    pages_out[:recall.size] = recall

    s_rng, w_rng, c_rng = streaming_regions(pos, sink, window)
    in_recall = np.zeros((pos // P + 1,), dtype=bool)   # candidates are <= pos
    in_recall[recall] = True
    cands = np.arange(c_rng.start, c_rng.stop, dtype=np.int64)
    cands = cands[in_recall[cands // P]]
    fixed = list(s_rng) + list(w_rng)
    D = k - len(fixed)
    if cands.size:
        sc = indexer_scores_row(q_row, w_row, keys[cands], cands.size)
        dyn = top_by_score(cands, sc, D)
    else:
        dyn = np.zeros((0,), np.int64)
    sel = np.concatenate([np.asarray(fixed, np.int64), dyn])
    idx[:sel.size] = sel
    return idx, pages_out


def index_hier(q, w, k, page_keys, seq_len, *, P: int, M: int, budget: int,
               sink: int, window: int, rows: Optional[list] = None):
    """Batch form. q [B,T,H,d], w [B,T,H], k [B,L_max,d], page_keys [B,L_max//P,d]
    (bf16 codes). Returns (idx [B,T,k], pages [B,T,M])."""
    B, T, H, d = q.shape
    L_max = k.shape[1]
    idx = np.full((B, T, budget), -1, dtype=np.int32)
    pages = np.full((B, T, M), -1, dtype=np.int32)
    todo = rows if rows is not None else [(b, t) for b in range(B) for t in range(T)]
    by_b = {}
    for b, t in todo:
        by_b.setdefault(b, []).append(t)
    for b, ts in by_b.items():
        L = int(min(max(int(seq_len[b]), 0), L_max))
        kd = bf16_to_f64(k[b, :L])
        pk = bf16_to_f64(page_keys[b, :L // P])
        for t in ts:
            pos = L - T + t
            idx[b, t], pages[b, t] = index_hier_row(
                bf16_to_f64(q[b, t]), np.asarray(w[b, t], np.float64), kd, pk,
                pos, P, M, budget, sink, window)
    return idx, pages


def pool_pages_e4m3(k8: np.ndarray, k_scale: np.ndarray, seq_len: np.ndarray, P: int):
    """Page keys from e4m3 token keys (R12): k8 [B, L_max, d] codes with
    k_scale [B, L_max] -> (page codes [B, L_max // P, d], page scales [B, L_max // P]).
    Pages that are not full are returned as code 0 with scale 1."""
    B, L_max, d = k8.shape
    n_pages = L_max // P
    codes = np.zeros((B, n_pages, d), dtype=np.uint8)
    scales = np.ones((B, n_pages), dtype=np.float32)
    for b in range(B):
        L = int(min(max(int(seq_len[b]), 0), L_max))
        n_full = L // P
        if n_full == 0:
            continue
        x = (e4m3_to_f64(k8[b, :n_full * P]).astype(np.float32) *
             np.asarray(k_scale[b, :n_full * P], np.float32)[:, None]).astype(np.float32)
        x = x.reshape(n_full, P, d)
        acc = np.zeros((n_full, d), dtype=np.float32)
        for j in range(P):                      # float32 adds, ascending row order
            acc = (acc + x[:, j, :]).astype(np.float32)
        mean = (acc / np.float32(P)).astype(np.float32)
        amax = np.max(np.abs(mean), axis=1)
        sc = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
        codes[b, :n_full] = f64_to_e4m3_rne((mean / sc[:, None]).astype(np.float32))
        scales[b, :n_full] = sc
    return codes, scales


def index_hier_e4m3(q8, q_scale, w, k8, k_scale, page_codes, page_scales, seq_len, *, P: int,
                    M: int, budget: int, sink: int, window: int):
    """FP8 hierarchical indexing (R12): R7 on dequantized queries, token keys and
    page keys. Returns (idx [B,T,k], pages [B,T,M])."""
    B, T = q8.shape[0], q8.shape[1]
    L_max = k8.shape[1]
    idx = np.full((B, T, budget), -1, dtype=np.int32)
    pages = np.full((B, T, M), -1, dtype=np.int32)
    for b in range(B):
        L = int(min(max(int(seq_len[b]), 0), L_max))
        kd = _decode_k(k8[b, :L], k_scale[b, :L], True)
        pk = _decode_k(page_codes[b, :L // P], page_scales[b, :L // P], True)
        for t in range(T):
            idx[b, t], pages[b, t] = index_hier_row(
                _decode_q(q8[b, t], q_scale[b, t], True), np.asarray(w[b, t], np.float64), kd, pk,
                L - T + t, P, M, budget, sink, window)
    return idx, pages


# ---------------------------------------------------------------------------
# Compressed-entry indexing (DSA article, "Technical Evolution and
# Applications": top-k over compressed historical entries; R11)
# ---------------------------------------------------------------------------


def entry_position(pos: int, m: int) -> int:
    """Position of the query at token ``pos`` among entries of ``m`` tokens: the
    last complete entry, -1 if none is complete yet (R11)."""
    return (pos + 1) // m - 1


def index_compressed(q, w, entry_keys, seq_len, *, m: int, budget: int, sink: int,
                     window: int, q_scale=None, k_scale=None, fp8: bool = False):
    """Indexing over compressed entries. entry_keys [B, L_max // m, d] (bf16 or
    e4m3 codes); seq_len in tokens. Returns (idx [B,T,budget] entry ids, scores
    float32 [B,T,L_max // m] with -inf at entries not yet complete)."""
    B, T = q.shape[0], q.shape[1]
    n_e = entry_keys.shape[1]
    L_max = n_e * m
    scores = np.full((B, T, n_e), NEG_INF32, dtype=np.float32)
    idx = np.full((B, T, budget), -1, dtype=np.int32)
    for b in range(B):
        L = int(min(max(int(seq_len[b]), 0), L_max))
        kd = _decode_k(entry_keys[b], None if k_scale is None else k_scale[b], fp8)
        for t in range(T):
            pe = entry_position(L - T + t, m)
            if pe < 0:
                continue
            qd = _decode_q(q[b, t], None if q_scale is None else q_scale[b, t], fp8)
            scores[b, t] = indexer_scores_row(qd, np.asarray(w[b, t], np.float64), kd, pe + 1)
            idx[b, t] = select_streaming_row(scores[b, t], pe, budget, sink, window)
    return idx, scores


# ---------------------------------------------------------------------------
# Sparse attention (article: "Sparse Attention Calculator"; LSA abstract:
# attention reads only the selected KV entries; R8)
# ---------------------------------------------------------------------------


def sparse_attention_row(qa: np.ndarray, k_rows: np.ndarray, v_rows: np.ndarray,
                         idx: np.ndarray, scale: float):
    """One query: qa float64 [Hq, d_qk]; k_rows / v_rows float64 [L, *] (this
    sequence's cache); idx int [k] with -1 padding. Returns (o [Hq, d_v] float64,
    lse [Hq] float64)."""
    Hq = qa.shape[0]
    d_v = v_rows.shape[1]
    valid = np.asarray(idx)[np.asarray(idx) >= 0].astype(np.int64)
    if valid.size == 0:
        return np.zeros((Hq, d_v)), np.full((Hq,), -np.inf)
    K = k_rows[valid]
    V = v_rows[valid]
    logits = scale * (qa @ K.T)                       # [Hq, n]
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ V) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def sparse_attention(qa, idx, seq_len, *, scale: float, d_v: int, kv=None, k=None,
                     v=None, rows: Optional[list] = None):
    """Batch form. qa [B,T,Hq,d_qk] bf16; idx [B,T,k]; either ``kv`` [B,L_max,d_qk]
    (MLA: V = kv[..., :d_v]) or separate ``k`` [B,L_max,d_qk] and ``v``
    [B,L_max,d_v]. Returns (o [B,T,Hq,d_v] float64, lse [B,T,Hq] float64).

    Only rows of the cache that some index names are decoded."""
    B, T, Hq, d_qk = qa.shape
    o = np.zeros((B, T, Hq, d_v))
    lse = np.full((B, T, Hq), -np.inf)
    todo = rows if rows is not None else [(b, t) for b in range(B) for t in range(T)]
    for b, t in todo:
        sel = np.asarray(idx[b, t])
        valid = np.unique(sel[sel >= 0]).astype(np.int64)
        if valid.size == 0:
            continue
        remap = np.full((int(valid.max()) + 1,), -1, dtype=np.int64)
        remap[valid] = np.arange(valid.size)
        local = np.where(sel >= 0, remap[np.maximum(sel, 0)], -1)
        if kv is not None:
            Kr = bf16_to_f64(kv[b, valid, :d_qk])
            Vr = bf16_to_f64(kv[b, valid, :d_v])
        else:
            Kr = bf16_to_f64(k[b, valid, :d_qk])
            Vr = bf16_to_f64(v[b, valid, :d_v])
        o[b, t], lse[b, t] = sparse_attention_row(bf16_to_f64(qa[b, t]), Kr, Vr, local, scale)
    return o, lse


# ---------------------------------------------------------------------------
# Cross-layer group (LSA abstract (2); key contributions: indexing cost 1/N;
# model card "CLI"; R9)
# ---------------------------------------------------------------------------


def layer_group(q, w, k, seq_len, layers, *, budget: int, sink: int, window: int,
                P: int = 0, M: int = 0, page_keys=None):
    """One indexing pass (flat if P == 0, else hierarchical) feeding every layer.

    ``layers`` is a list of dicts with keys qa, scale, d_v and either kv or k/v.
    Returns (idx, [ (o, lse) per layer ])."""
    if P:
        idx, _ = index_hier(q, w, k, page_keys, seq_len, P=P, M=M, budget=budget,
                            sink=sink, window=window)
    else:
        idx, _ = index_flat(q, w, k, seq_len, budget=budget, sink=sink, window=window)
    outs = []
    for lay in layers:
        outs.append(sparse_attention(lay["qa"], idx, seq_len, scale=lay["scale"],
                                     d_v=lay["d_v"], kv=lay.get("kv"), k=lay.get("k"),
                                     v=lay.get("v")))
    return idx, outs
