"""CPU oracle of the LSA hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
may import this package. The product path never does, and the oracle shares no
code with the CUDA library.

The oracle is the plain C++ in ``oracle/lsa_oracle.cpp`` (built into
``oracle/liblsa_oracle.so`` by ``oracle/build.py``, on first use if needed).
This module only marshals numpy arrays into its C entry points: every score,
selection, pooling and attention value comes from the C++ code. The functions
keep the names and signatures the tests use; see the C++ source for the
readings (R1-R12) of the pages that each step follows.

``oracle/numpy_oracle.py`` is a second, independent restatement of the same
definitions with numpy/BLAS, kept only as a cross-check of this one
(``tests/test_oracle_cross_check.py``).

Threads: the C++ harness runs independent rows (or key chunks of a row) on
``threads()`` host cores; ``set_threads(n)`` changes it (0 = every core this
process may use). The arithmetic of a row does not depend on the thread count.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np

from . import build as _build

NEG_INF32 = np.float32(-np.inf)

_lib = None
_threads = 0


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        c = ctypes
        P, i32, i64, f64 = c.c_void_p, c.c_int, c.c_int64, c.c_double
        sig = {
            "orc_host_threads": (i32, []),
            "orc_bf16_to_f64": (None, [i64, P, P]),
            "orc_f32_to_bf16_rne": (None, [i64, P, P]),
            "orc_e4m3_to_f64": (None, [i64, P, P]),
            "orc_f64_to_e4m3_rne": (None, [i64, P, P]),
            "orc_indexer_scores_row": (i32, [P, P, P, i32, i32, i64, i64, P]),
            "orc_indexer_scores_rows": (i32, [i32, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, i32, P,
                                              i32]),
            "orc_streaming_regions": (None, [i64, i64, i64, P]),
            "orc_select_row": (i32, [P, i64, i64, i32, i32, i32, P]),
            "orc_select_streaming": (i32, [P, P, i32, i32, i32, i32, i32, i32, P, i32]),
            "orc_page_sets": (i32, [i64, i64, i64, i64, P, i32, P]),
            "orc_pool_pages": (i32, [P, P, i32, i32, i32, i32, P]),
            "orc_pool_pages_e4m3": (i32, [P, P, P, i32, i32, i32, i32, P, P]),
            "orc_index_hier_row": (i32, [P, P, i32, i32, P, i64, P, i64, i64, i32, i32, i32, i32, i32, P, P]),
            "orc_index_hier": (i32, [i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                     P, i32, P, P, i32]),
            "orc_index_compressed": (i32, [i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, i32, i32, i32, P, P,
                                           i32]),
            "orc_sparse_attention_row": (i32, [P, P, P, i64, i32, i32, i32, P, i64, f64, P, P]),
            "orc_sparse_attention": (i32, [i32, i32, i32, i32, i32, i32, P, P, i32, P, i64, P, i64, f64, P, i32, P,
                                           P, i32]),
            "orc_sparse_attention_e4m3": (i32, [i32, i32, i32, i32, i32, i32, P, P, i32, P, i64, P, f64, P, i32, P,
                                                P, i32]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def set_threads(n: int) -> None:
    """Host threads for the oracle's row harness (0 = every available core)."""
    global _threads
    _threads = int(n)


def threads() -> int:
    """Threads the harness uses: set_threads()'s value, else every available core."""
    return _threads if _threads > 0 else int(_load().orc_host_threads())


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _ok(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected its arguments")


def _rows_arg(rows, B, T):
    if rows is None:
        return None, B * T
    r = _c(np.asarray(rows, dtype=np.int64).reshape(-1, 2), np.int32)
    return r, r.shape[0]


# ---------------------------------------------------------------------------
# element codecs
# ---------------------------------------------------------------------------


def bf16_to_f64(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64."""
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    _load().orc_bf16_to_f64(b.size, _p(b), _p(out))
    return out


def f32_to_bf16_rne(x) -> np.ndarray:
    """float32 -> bf16 bit pattern, round to nearest even; NaN stays NaN."""
    a = _c(x, np.float32)
    out = np.empty(a.shape, np.uint16)
    _load().orc_f32_to_bf16_rne(a.size, _p(a), _p(out))
    return out


def e4m3_to_f64(codes) -> np.ndarray:
    """OCP FP8 E4M3 code -> float64 (NaN for the two NaN codes)."""
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().orc_e4m3_to_f64(c.size, _p(c), _p(out))
    return out


def f64_to_e4m3_rne(x) -> np.ndarray:
    """Real value -> nearest finite e4m3 code (ties to even code, saturating at 448)."""
    a = _c(x, np.float64)
    out = np.empty(a.shape, np.uint8)
    _load().orc_f64_to_e4m3_rne(a.size, _p(a), _p(out))
    return out


# ---------------------------------------------------------------------------
# indexer scores
# ---------------------------------------------------------------------------


def indexer_scores_row(q_row, w_row, keys, n_visible: int) -> np.ndarray:
    """Scores of one float64 query [H, d] (weights [H]) against float64 keys
    [n, d]; keys at or beyond n_visible get -inf. Returns float32 [n]."""
    q, w, k = _c(q_row, np.float64), _c(w_row, np.float64), _c(keys, np.float64)
    n, d = k.shape
    out = np.empty((n,), np.float32)
    _ok(_load().orc_indexer_scores_row(_p(q), _p(w), _p(k), q.shape[0], d, n, int(n_visible), _p(out)),
        "indexer_scores_row")
    return out


def _indexer_args(q, w, k, q_scale, k_scale, fp8):
    if fp8:
        return (_c(q, np.uint8), _c(q_scale, np.float32), _c(w, np.float32), _c(k, np.uint8),
                _c(k_scale, np.float32))
    return _c(q, np.uint16), None, _c(w, np.float32), _c(k, np.uint16), None


def indexer_scores_rows(q, w, k, seq_len, rows, *, q_scale=None, k_scale=None, fp8: bool = False,
                        vis_shift: int = 0, L_max: Optional[int] = None) -> np.ndarray:
    """Flat indexer scores of the listed (b, t) rows, compact: float32
    [len(rows), keys per sequence]. q [B,T,H,d], w [B,T,H], k [B,n,d] (bf16
    codes, or e4m3 codes with q_scale [B,T,H] / k_scale [B,n]). Key s is visible
    iff s < (pos + 1) >> vis_shift (vis_shift = log2 m for compressed entries,
    whose seq_len and L_max count tokens)."""
    qq, qs, ww, kk, ks = _indexer_args(q, w, k, q_scale, k_scale, fp8)
    B, T, H, d = qq.shape
    n_keys = kk.shape[1]
    sl = _c(seq_len, np.int32)
    r, n = _rows_arg(rows, B, T)
    out = np.empty((n, n_keys), np.float32)
    _ok(_load().orc_indexer_scores_rows(B, T, H, d, n_keys, n_keys << vis_shift if L_max is None else L_max,
                                        vis_shift, int(bool(fp8)), _p(qq), _p(qs), _p(ww), _p(kk), _p(ks), _p(sl),
                                        _p(r), n, _p(out), _threads), "indexer_scores_rows")
    return out


def indexer_scores(q, w, k, seq_len, *, q_scale=None, k_scale=None, fp8: bool = False,
                   rows: Optional[list] = None) -> np.ndarray:
    """Flat indexer scores for a batch: float32 [B,T,L_max], -inf at invisible
    slots. ``rows`` restricts the work to a list of (b, t); other rows stay -inf."""
    B, T = np.shape(q)[:2]
    L_max = np.shape(k)[1]
    if rows is None:
        return indexer_scores_rows(q, w, k, seq_len, None, q_scale=q_scale, k_scale=k_scale,
                                   fp8=fp8).reshape(B, T, L_max)
    out = np.full((B, T, L_max), NEG_INF32, dtype=np.float32)
    got = indexer_scores_rows(q, w, k, seq_len, rows, q_scale=q_scale, k_scale=k_scale, fp8=fp8)
    for i, (b, t) in enumerate(rows):
        out[b, t] = got[i]
    return out


# ---------------------------------------------------------------------------
# streaming selection
# ---------------------------------------------------------------------------


def streaming_regions(pos: int, sink: int, window: int):
    """(sink, window, dynamic-candidate) token ranges of a query at ``pos``."""
    out = np.zeros(3, np.int64)
    _load().orc_streaming_regions(int(pos), int(sink), int(window), _p(out))
    se, wl, wh = (int(v) for v in out)
    return range(0, se), range(wl, wh), range(se, wl)


def select_streaming_row(scores, pos: int, k: int, sink: int, window: int) -> np.ndarray:
    """Index row of one query from its float32 scores (-inf = not a candidate)."""
    s = _c(scores, np.float32)
    out = np.empty((k,), np.int32)
    _ok(_load().orc_select_row(_p(s), s.size, int(pos), int(k), int(sink), int(window), _p(out)),
        "select_streaming_row")
    return out


def select_streaming(scores, seq_len, T: int, k: int, sink: int, window: int) -> np.ndarray:
    """scores [B,T,L_max] float32 -> idx [B,T,k] int32."""
    s = _c(scores, np.float32)
    B, _, L_max = s.shape
    sl = _c(seq_len, np.int32)
    out = np.empty((B, T, k), np.int32)
    _ok(_load().orc_select_streaming(_p(s), _p(sl), B, int(T), L_max, int(k), int(sink), int(window), _p(out),
                                     _threads), "select_streaming")
    return out


def index_flat(q, w, k, seq_len, *, budget: int, sink: int, window: int, q_scale=None, k_scale=None,
               fp8: bool = False):
    """Flat indexing: scores, then the streaming selection. Returns (idx, scores)."""
    sc = indexer_scores(q, w, k, seq_len, q_scale=q_scale, k_scale=k_scale, fp8=fp8)
    return select_streaming(sc, seq_len, np.shape(q)[1], budget, sink, window), sc


# ---------------------------------------------------------------------------
# hierarchical indexing
# ---------------------------------------------------------------------------


def pool_pages(k_bits, seq_len, P: int) -> np.ndarray:
    """Mean-pooled bf16 page keys [B, L_max // P, d]; pages not full are 0."""
    k = _c(k_bits, np.uint16)
    B, L_max, d = k.shape
    out = np.empty((B, L_max // P, d), np.uint16)
    _ok(_load().orc_pool_pages(_p(k), _p(_c(seq_len, np.int32)), B, L_max, d, int(P), _p(out)), "pool_pages")
    return out


def pool_pages_e4m3(k8, k_scale, seq_len, P: int):
    """Page keys from e4m3 token keys: (codes [B, L_max // P, d], scales [B, L_max // P])."""
    k = _c(k8, np.uint8)
    B, L_max, d = k.shape
    codes = np.empty((B, L_max // P, d), np.uint8)
    scales = np.empty((B, L_max // P), np.float32)
    _ok(_load().orc_pool_pages_e4m3(_p(k), _p(_c(k_scale, np.float32)), _p(_c(seq_len, np.int32)), B, L_max, d,
                                    int(P), _p(codes), _p(scales)), "pool_pages_e4m3")
    return codes, scales


def page_sets(pos: int, P: int, sink: int, window: int):
    """Forced pages (sorted list) and the eligible page range of a query at ``pos``."""
    cap = (int(sink) + P - 1) // P + (int(window) + P - 1) // P + 2
    forced = np.zeros(cap, np.int64)
    er = np.zeros(2, np.int64)
    n = _load().orc_page_sets(int(pos), int(P), int(sink), int(window), _p(forced), cap, _p(er))
    _ok(0 if n >= 0 else -1, "page_sets")
    return [int(v) for v in forced[:n]], range(int(er[0]), int(er[1]))


def index_hier_row(q_row, w_row, keys, page_keys, pos: int, P: int, M: int, k: int, sink: int, window: int):
    """Coarse-to-fine selection of one float64 query: keys [L, d] (this sequence),
    page_keys [n_pages, d]. Returns (idx [k], pages [M] ascending, -1 padded)."""
    q, w = _c(q_row, np.float64), _c(w_row, np.float64)
    kk, pk = _c(keys, np.float64), _c(page_keys, np.float64)
    idx = np.empty((k,), np.int32)
    pages = np.empty((M,), np.int32)
    _ok(_load().orc_index_hier_row(_p(q), _p(w), q.shape[0], q.shape[1], _p(kk), kk.shape[0], _p(pk), pk.shape[0],
                                   int(pos), int(P), int(M), int(k), int(sink), int(window), _p(idx), _p(pages)),
        "index_hier_row")
    return idx, pages


def _index_hier(q, q_scale, w, k, k_scale, page_keys, page_scales, seq_len, fp8, P, M, budget, sink, window, rows):
    qq, qs, ww, kk, ks = _indexer_args(q, w, k, q_scale, k_scale, fp8)
    pk = _c(page_keys, np.uint8 if fp8 else np.uint16)
    ps = _c(page_scales, np.float32) if fp8 else None
    B, T, H, d = qq.shape
    L_max = kk.shape[1]
    r, n = _rows_arg(rows, B, T)
    idx = np.empty((n, budget), np.int32)
    pages = np.empty((n, M), np.int32)
    _ok(_load().orc_index_hier(B, T, H, d, L_max, int(bool(fp8)), _p(qq), _p(qs), _p(ww), _p(kk), _p(ks), _p(pk),
                               _p(ps), _p(_c(seq_len, np.int32)), int(P), int(M), int(budget), int(sink), int(window),
                               _p(r), n, _p(idx), _p(pages), _threads), "index_hier")
    if rows is None:
        return idx.reshape(B, T, budget), pages.reshape(B, T, M)
    full_i = np.full((B, T, budget), -1, np.int32)
    full_p = np.full((B, T, M), -1, np.int32)
    for i, (b, t) in enumerate(rows):
        full_i[b, t], full_p[b, t] = idx[i], pages[i]
    return full_i, full_p


def index_hier(q, w, k, page_keys, seq_len, *, P: int, M: int, budget: int, sink: int, window: int,
               rows: Optional[list] = None):
    """bf16 hierarchical indexing. Returns (idx [B,T,k], pages [B,T,M])."""
    return _index_hier(q, None, w, k, None, page_keys, None, seq_len, False, P, M, budget, sink, window, rows)


def index_hier_e4m3(q8, q_scale, w, k8, k_scale, page_codes, page_scales, seq_len, *, P: int, M: int, budget: int,
                    sink: int, window: int, rows: Optional[list] = None):
    """FP8 hierarchical indexing on dequantized queries, token and page keys."""
    return _index_hier(q8, q_scale, w, k8, k_scale, page_codes, page_scales, seq_len, True, P, M, budget, sink,
                       window, rows)


# ---------------------------------------------------------------------------
# compressed entries
# ---------------------------------------------------------------------------


def entry_position(pos: int, m: int) -> int:
    """The last complete entry of m tokens for a query at token ``pos`` (-1: none)."""
    return (int(pos) + 1) // int(m) - 1


def index_compressed(q, w, entry_keys, seq_len, *, m: int, budget: int, sink: int, window: int, q_scale=None,
                     k_scale=None, fp8: bool = False):
    """Indexing over compressed entries: entry_keys [B, L_max // m, d]; seq_len in
    tokens. Returns (idx [B,T,budget] entry ids, scores float32 [B,T,L_max // m])."""
    qq, qs, ww, kk, ks = _indexer_args(q, w, entry_keys, q_scale, k_scale, fp8)
    B, T, H, d = qq.shape
    n_e = kk.shape[1]
    scores = np.empty((B, T, n_e), np.float32)
    idx = np.empty((B, T, budget), np.int32)
    _ok(_load().orc_index_compressed(B, T, H, d, n_e, int(m), int(bool(fp8)), _p(qq), _p(qs), _p(ww), _p(kk), _p(ks),
                                     _p(_c(seq_len, np.int32)), int(budget), int(sink), int(window), _p(scores),
                                     _p(idx), _threads), "index_compressed")
    return idx, scores


# ---------------------------------------------------------------------------
# sparse attention
# ---------------------------------------------------------------------------


def sparse_attention_row(qa, k_rows, v_rows, idx, scale: float):
    """One float64 query [Hq, d_qk] over float64 K [n, d_qk] / V [n, d_v] rows of
    its sequence, indices idx (-1 skipped). Returns (o [Hq, d_v], lse [Hq])."""
    q, K, V = _c(qa, np.float64), _c(k_rows, np.float64), _c(v_rows, np.float64)
    ix = _c(idx, np.int64)
    Hq, d_qk = q.shape
    d_v = V.shape[1]
    o = np.empty((Hq, d_v), np.float64)
    lse = np.empty((Hq,), np.float64)
    _ok(_load().orc_sparse_attention_row(_p(q), _p(K), _p(V), K.shape[0], Hq, d_qk, d_v, _p(ix), ix.size,
                                         float(scale), _p(o), _p(lse)), "sparse_attention_row")
    return o, lse


def sparse_attention_rows(qa, idx, rows, *, scale: float, d_v: int, kv=None, k=None, v=None):
    """Attention of the listed (b, t) rows (None = all), compact: (o [n, Hq, d_v],
    lse [n, Hq]) in float64. qa [B,T,Hq,d_qk] bf16; idx [B,T,kk]; MLA ``kv``
    [B,L_max,d_qk] (V = its first d_v columns) or separate ``k``, ``v``."""
    q = _c(qa, np.uint16)
    B, T, Hq, d_qk = q.shape
    ix = _c(idx, np.int32)
    if kv is not None:
        kk = vv = _c(kv, np.uint16)
    else:
        kk, vv = _c(k, np.uint16), _c(v, np.uint16)
    L_max = kk.shape[1]
    r, n = _rows_arg(rows, B, T)
    o = np.empty((n, Hq, d_v), np.float64)
    lse = np.empty((n, Hq), np.float64)
    _ok(_load().orc_sparse_attention(B, T, Hq, d_qk, d_v, L_max, _p(q), _p(ix), ix.shape[2], _p(kk), kk.shape[2],
                                     _p(vv), vv.shape[2], float(scale), _p(r), n, _p(o), _p(lse), _threads),
        "sparse_attention")
    return o, lse


def sparse_attention_e4m3_rows(qa, idx, rows, *, scale: float, d_v: int, kv8, k_scale):
    """Attention over an e4m3 latent cache (K = code * scale, V = its first d_v
    columns), for the listed (b, t) rows (None = all), compact: (o [n, Hq, d_v],
    lse [n, Hq]) in float64. kv8 [B,L_max,d_qk] e4m3 codes; k_scale [B,L_max] fp32."""
    q = _c(qa, np.uint16)
    B, T, Hq, d_qk = q.shape
    ix = _c(idx, np.int32)
    kc = _c(kv8, np.uint8)
    ks = _c(k_scale, np.float32)
    L_max = kc.shape[1]
    if ks.shape != (kc.shape[0], L_max):
        raise ValueError("k_scale must be [B, L_max]")
    r, n = _rows_arg(rows, B, T)
    o = np.empty((n, Hq, d_v), np.float64)
    lse = np.empty((n, Hq), np.float64)
    _ok(_load().orc_sparse_attention_e4m3(B, T, Hq, d_qk, d_v, L_max, _p(q), _p(ix), ix.shape[2], _p(kc), kc.shape[2],
                                          _p(ks), float(scale), _p(r), n, _p(o), _p(lse), _threads),
        "sparse_attention_e4m3")
    return o, lse


def sparse_attention(qa, idx, seq_len, *, scale: float, d_v: int, kv=None, k=None, v=None,
                     rows: Optional[list] = None):
    """Batch form: (o [B,T,Hq,d_v], lse [B,T,Hq]) in float64; rows not listed stay
    0 / -inf. seq_len is not needed (the index rows name the keys)."""
    B, T, Hq = np.shape(qa)[:3]
    o, lse = sparse_attention_rows(qa, idx, rows, scale=scale, d_v=d_v, kv=kv, k=k, v=v)
    if rows is None:
        return o.reshape(B, T, Hq, d_v), lse.reshape(B, T, Hq)
    fo = np.zeros((B, T, Hq, d_v))
    fl = np.full((B, T, Hq), -np.inf)
    for i, (b, t) in enumerate(rows):
        fo[b, t], fl[b, t] = o[i], lse[i]
    return fo, fl


# ---------------------------------------------------------------------------
# cross-layer group (composition of the calls above, R9)
# ---------------------------------------------------------------------------


def layer_group(q, w, k, seq_len, layers, *, budget: int, sink: int, window: int, P: int = 0, M: int = 0,
                page_keys=None):
    """One indexing pass (flat if P == 0, else hierarchical) feeding every layer.
    ``layers``: dicts with qa, scale, d_v and kv (MLA) or k/v.
    Returns (idx, [(o, lse) per layer])."""
    if P:
        idx, _ = index_hier(q, w, k, page_keys, seq_len, P=P, M=M, budget=budget, sink=sink, window=window)
    else:
        idx, _ = index_flat(q, w, k, seq_len, budget=budget, sink=sink, window=window)
    outs = [sparse_attention(lay["qa"], idx, seq_len, scale=lay["scale"], d_v=lay["d_v"], kv=lay.get("kv"),
                             k=lay.get("k"), v=lay.get("v")) for lay in layers]
    return idx, outs
