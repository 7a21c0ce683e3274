"""The index-row parity check rejects every kind of invalid row (no GPU).

Mistakes are planted in oracle rows on the CPU; each must trip
tests.parity.check_index_row, while the oracle row itself and a genuine
near-tie swap pass.
"""
import numpy as np
import pytest

import oracle as O
from kv_indexing_b200 import inputs as I
from tests.parity import check_index_row

W = I.Workload(name="pc", B=1, L=600, T=1, H=4, d=64, k=96, sink=8, window=24, needles=12)
POS = W.L - 1


@pytest.fixture(scope="module")
def row():
    x = I.make_indexer_inputs(W, 11)
    idx, sc = O.index_flat(x["q_idx"], x["w"], x["k_idx"], x["seq_len"], budget=W.k, sink=W.sink, window=W.window)
    return idx[0, 0].copy(), sc[0, 0].copy()


def check(g, o, sc):
    return check_index_row(g, o, sc, POS, W.sink, W.window)


def test_oracle_row_passes(row):
    o, sc = row
    assert check(o.copy(), o, sc) == 0


@pytest.mark.parametrize("plant", ["window_repeat", "sink_repeat", "beyond_pos", "hole", "short", "unsorted",
                                   "far_swap", "lead_changed"])
def test_planted_mistakes_fail(row, plant):
    o, sc = row
    g = o.copy()
    lead = W.sink + W.window
    if plant == "window_repeat":          # a window token repeated in the dynamic block
        g[lead] = POS - 1
        g[lead:np.sum(g >= 0)] = np.sort(g[lead:np.sum(g >= 0)])
    elif plant == "sink_repeat":          # a sink token repeated in the dynamic block
        g[lead] = 3
        g[lead:np.sum(g >= 0)] = np.sort(g[lead:np.sum(g >= 0)])
    elif plant == "beyond_pos":
        g[np.sum(g >= 0) - 1] = POS + 5
    elif plant == "hole":                 # -1 in the middle of the valid entries
        g[lead + 3] = -1
    elif plant == "short":                # one valid entry dropped
        g[np.sum(g >= 0) - 1] = -1
    elif plant == "unsorted":
        g[lead], g[lead + 1] = g[lead + 1], g[lead]
    elif plant == "far_swap":             # the lowest candidate swapped for one far below the threshold
        dyn = o[lead:np.sum(o >= 0)]
        cand = np.arange(W.sink, POS - W.window + 1)
        out = np.setdiff1d(cand, dyn)
        worst = out[np.argmin(sc[out])]
        keep = np.setdiff1d(dyn, [dyn[np.argmin(sc[dyn])]])
        g[lead:np.sum(o >= 0)] = np.sort(np.append(keep, worst))
    elif plant == "lead_changed":
        g[0] = 1
    with pytest.raises(AssertionError):
        check(g, o, sc)


def test_near_tie_swap_passes(row):
    o, sc = row
    sc = sc.copy()
    lead = W.sink + W.window
    dyn = o[lead:np.sum(o >= 0)]
    cand = np.arange(W.sink, POS - W.window + 1)
    out = np.setdiff1d(cand, dyn)
    tau = sc[dyn].min()
    sc[out[0]] = tau * np.float32(1 - 1e-4)        # an outsider within 1e-3 of the threshold
    g = o.copy()
    keep = np.setdiff1d(dyn, [dyn[np.argmin(sc[dyn])]])
    g[lead:np.sum(o >= 0)] = np.sort(np.append(keep, out[0]))
    assert check(g, o, sc) == 1
