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


def check_index_row(g, o, scores, n_lead, tol=TIE_RTOL):
    """GPU index row g vs oracle row o (both canonical). The first n_lead entries
    (sink + window) must match exactly; the dynamic blocks may differ only by swaps
    among candidates whose oracle score lies within tol (relative) of the oracle's
    D-th selected score. Returns the number of swapped pairs."""
    g = np.asarray(g)
    o = np.asarray(o)
    assert np.array_equal(g[:n_lead], o[:n_lead]), "sink/window block differs"
    gv, ov = g[g >= 0], o[o >= 0]
    assert gv.size == ov.size, f"valid counts differ: {gv.size} vs {ov.size}"
    gd, od = gv[n_lead:], ov[n_lead:]
    assert np.all(np.diff(gd) > 0), "dynamic block not strictly ascending"
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


def lead_count(pos, sink, window):
    s, w, _ = O.streaming_regions(pos, sink, window)
    return len(s) + len(w)


def assert_attention_close(g, o):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    err = np.abs(g - o)
    mx = float(err.max()) if err.size else 0.0
    rel = mx / max(float(np.abs(o).max()), 1e-30) if err.size else 0.0
    assert mx <= ATTN_ATOL, f"attention max-abs error {mx:.3g}"
    assert rel <= ATTN_RTOL, f"attention relative error {rel:.3g}"
    return mx, rel
