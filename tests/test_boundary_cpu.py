"""C-ABI boundary checks that need no GPU: the library loads, exports every
function include/lsa.h declares, and rejects bad arguments on the host before
touching the device."""
import ctypes
import os
import re

import pytest

from kv_indexing_b200 import lsa as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "lsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ["lsa_index_flat", "lsa_index_hier", "lsa_select_streaming", "lsa_sparse_attn",
                 "lsa_layer_group", "lsa_pool_pages", "lsa_workspace_size", "lsa_status_string"]:
        assert name in fns
    assert sorted(L.EXPORTS) == fns


def test_library_exports_every_declared_symbol():
    lib = L.load()
    for name in header_functions():
        assert hasattr(lib, name), name
    raw = ctypes.CDLL(L.LIB_PATH)
    for name in header_functions():
        getattr(raw, name)


def test_status_strings():
    lib = L.load()
    for st in range(6):
        assert lib.lsa_status_string(st)
    assert lib.lsa_status_string(99) == b"unknown status"


def _indexer(**kw):
    base = dict(B=1, T=1, H=64, d=128, L_max=1024, dtype=L.LSA_BF16, seq_len=16, q=32, q_scale=None, w=48, k=64,
                k_scale=None)
    base.update(kw)
    return L.IndexerIn(*[base[f] for f, _ in L.IndexerIn._fields_])


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), L.LSA_ERR_INVALID_ARG),
    (dict(d=96), L.LSA_ERR_UNSUPPORTED),
    (dict(H=6), L.LSA_ERR_UNSUPPORTED),
    (dict(L_max=1000), L.LSA_ERR_UNSUPPORTED),
    (dict(q=None), L.LSA_ERR_INVALID_ARG),
    (dict(k=72), L.LSA_ERR_INVALID_ARG),              # misaligned pointer
    (dict(dtype=L.LSA_E4M3), L.LSA_ERR_INVALID_ARG),  # e4m3 without scales
    (dict(dtype=L.LSA_E4M3, q_scale=16, k_scale=16, d=64), L.LSA_ERR_UNSUPPORTED),
])
def test_index_flat_rejects_bad_indexer_on_host(kw, code):
    lib = L.load()
    ii = _indexer(**kw)
    st = lib.lsa_index_flat(ctypes.byref(ii), L.Budget(2048, 64, 960), 16, None, None, 0, None)
    assert st == code, lib.lsa_last_error()
    assert lib.lsa_last_error()


@pytest.mark.parametrize("budget,code", [
    ((0, 0, 0), L.LSA_ERR_UNSUPPORTED),
    ((100, 60, 60), L.LSA_ERR_INVALID_ARG),
    ((100, -1, 0), L.LSA_ERR_INVALID_ARG),
    ((9000, 0, 0), L.LSA_ERR_UNSUPPORTED),
])
def test_budget_validation(budget, code):
    lib = L.load()
    ii = _indexer()
    assert lib.lsa_index_flat(ctypes.byref(ii), L.Budget(*budget), 16, None, None, 0, None) == code


def test_workspace_checks_and_sizes():
    lib = L.load()
    ii = _indexer(B=8, T=1, L_max=131072)
    n = L.workspace_size(L.LSA_OP_INDEX_FLAT, indexer=ii, budget=(2048, 64, 960))
    n_ext = L.workspace_size(L.LSA_OP_INDEX_FLAT, indexer=ii, budget=(2048, 64, 960), scores_external=True)
    assert n - n_ext == 8 * 131072 * 4                     # the score buffer moves out of the workspace
    sel = L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=8, T=1, L_max=131072)
    assert sel == n_ext == 0                               # rows of <= 256K keys select in cluster shared memory
    st = lib.lsa_index_flat(ctypes.byref(ii), L.Budget(2048, 64, 960), 16, None, 256, n - 1, None)
    assert st == L.LSA_ERR_WORKSPACE
    big = L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=2, T=1, L_max=1 << 20)
    assert big > 0                                         # longer rows need selection scratch
    st = lib.lsa_select_streaming(16, 16, 2, 1, 1 << 20, L.Budget(2048, 64, 960), 16, 256, big - 1, None)
    assert st == L.LSA_ERR_WORKSPACE
    hi = L.workspace_size(L.LSA_OP_INDEX_HIER, indexer=_indexer(B=2, L_max=1 << 20), budget=(2048, 64, 960),
                          P=64, M=256)
    # page scores + recalled pages + fine scores, then the larger of the two selections' scratch
    sel_pages = L.workspace_size(L.LSA_OP_SELECT, budget=(256, 0, 0), B=2, T=1, L_max=1 << 14)
    sel_fine = L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=2, T=1, L_max=256 * 64)
    fixed = 2 * (1 << 14) * 4 + 2 * 256 * 4 + 2 * 256 * 64 * 4
    assert fixed <= hi <= fixed + max(sel_pages, sel_fine) + 256


def test_hier_e4m3_validation():
    lib = L.load()
    ii = _indexer(L_max=4096)
    ii.dtype = L.LSA_E4M3
    ii.q_scale, ii.k_scale = 1 << 20, 2 << 20
    bu = L.Budget(2048, 64, 960)
    # the bf16 entry point points e4m3 callers at the e4m3 one
    assert lib.lsa_index_hier(ctypes.byref(ii), 16, 64, 256, bu, 16, None, None, 0, None) == L.LSA_ERR_UNSUPPORTED
    assert b"lsa_index_hier_e4m3" in lib.lsa_last_error()
    assert lib.lsa_index_hier_e4m3(ctypes.byref(ii), 16, None, 64, 256, bu, 16, None, None, 0, None) \
        == L.LSA_ERR_INVALID_ARG                                  # page scales missing
    assert lib.lsa_pool_pages_e4m3(16, 16, 16, 1, 4096, 64, 64, 16, 16, None) == L.LSA_ERR_UNSUPPORTED   # d != 128
    assert lib.lsa_pool_pages_e4m3(16, 16, 16, 1, 4096, 128, 24, 16, 16, None) == L.LSA_ERR_UNSUPPORTED  # P
    # the workspace of the e4m3 call is the bf16 call's
    ii_bf = _indexer(L_max=4096)
    assert L.workspace_size(L.LSA_OP_INDEX_HIER, indexer=ii, budget=(2048, 64, 960), P=64, M=256) == \
        L.workspace_size(L.LSA_OP_INDEX_HIER, indexer=ii_bf, budget=(2048, 64, 960), P=64, M=256)


def test_hier_parameter_validation():
    lib = L.load()
    ii = _indexer(L_max=4096)
    bu = L.Budget(2048, 64, 960)
    assert lib.lsa_index_hier(ctypes.byref(ii), 16, 48, 256, bu, 16, None, None, 0, None) == L.LSA_ERR_UNSUPPORTED
    assert lib.lsa_index_hier(ctypes.byref(ii), 16, 64, 8, bu, 16, None, None, 0, None) == L.LSA_ERR_INVALID_ARG


def test_pool_and_select_validation():
    lib = L.load()
    assert lib.lsa_pool_pages(16, 16, 1, 4096, 128, 24, 16, None) == L.LSA_ERR_UNSUPPORTED
    assert lib.lsa_pool_pages(16, 16, 1, 4000, 128, 64, 16, None) == L.LSA_ERR_INVALID_ARG
    assert lib.lsa_select_streaming(None, 16, 1, 1, 128, L.Budget(8, 2, 2), 16, None, 0, None) == L.LSA_ERR_INVALID_ARG


def test_compressed_entry_validation_and_sizes():
    lib = L.load()
    bu = L.Budget(2048, 16, 240)
    for m in (3, 256, 0):
        ii = _indexer(L_max=4096)
        assert lib.lsa_index_compressed(ctypes.byref(ii), m, bu, 16, None, None, 0, None) == L.LSA_ERR_UNSUPPORTED
    ii = _indexer(L_max=4096)
    assert lib.lsa_index_compressed(ctypes.byref(ii), 4, bu, None, None, None, 0, None) == L.LSA_ERR_INVALID_ARG
    big = _indexer(B=4, L_max=1 << 20)
    n = L.workspace_size(L.LSA_OP_INDEX_COMPRESSED, indexer=big, budget=(2048, 16, 240), m=4)
    sel = L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 16, 240), B=4, T=1, L_max=1 << 18)
    assert n == 4 * (1 << 18) * 4 + sel    # entry scores + the selection's scratch over 262144-entry rows
    assert L.workspace_size(L.LSA_OP_INDEX_COMPRESSED, indexer=big, budget=(2048, 16, 240), m=4,
                            scores_external=True) == sel
    st = lib.lsa_index_compressed(ctypes.byref(big), 4, bu, 16, None, 256, n - 1, None)
    assert st == L.LSA_ERR_WORKSPACE


def test_selection_launch_shapes_by_workspace():
    # rows of <= 262144 slots: one cluster per row, keys in shared memory, no scratch
    assert L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=80, T=1, L_max=262144) == 0
    assert L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=4, T=1, L_max=262144) == 0
    # many longer rows: per-segment candidate lists in the workspace
    assert L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=80, T=1, L_max=262144 + 1025) > 0
    # few longer rows: the filter launch -- group maxima, a candidate pool of at
    # most D x G entries per row, per-warp tables, counters
    few = L.workspace_size(L.LSA_OP_SELECT, budget=(2048, 64, 960), B=4, T=1, L_max=1 << 20)
    assert 0 < few < 4 * (1 << 20) * 8


def _mla_layer(q, kv, B=1, T=1, L_max=1024, Hq=128):
    return L.AttnIn(B, T, Hq, 576, 512, L_max, 0.04, 16, q, kv, kv, 576, 576, -1, -1)


def test_layer_group_rejects_overlapping_outputs_on_host():
    lib = L.load()
    ii = _indexer(L_max=1024)
    layers = (L.AttnIn * 2)(_mla_layer(1 << 20, 2 << 20), _mla_layer(3 << 20, 4 << 20))
    bu = L.Budget(256, 16, 64)
    out_bytes = 1 * 1 * 128 * 512 * 2
    base = 64 << 20
    for o1 in (base, base + out_bytes - 256):        # the same buffer, then a partial overlap
        outs = (ctypes.c_void_p * 2)(base, o1)
        st = lib.lsa_layer_group(ctypes.byref(ii), None, 0, 0, bu, 2, layers, outs, None, None, None, 0, None)
        assert st == L.LSA_ERR_INVALID_ARG, lib.lsa_last_error()
        assert b"overlap" in lib.lsa_last_error()
    outs = (ctypes.c_void_p * 2)(base, base + out_bytes)
    idx_over = base + out_bytes + 512                  # idx inside the second layer's output
    st = lib.lsa_layer_group(ctypes.byref(ii), None, 0, 0, bu, 2, layers, outs, None, idx_over, None, 0, None)
    assert st == L.LSA_ERR_INVALID_ARG and b"idx" in lib.lsa_last_error()


def test_attention_e4m3_kv_validation():
    lib = L.load()
    idx = 5 << 20
    out = 6 << 20

    def call(**kw):
        ai = _mla_layer(1 << 20, 2 << 20)
        for f, v in kw.items():
            setattr(ai, f, v)
        return lib.lsa_sparse_attn(ctypes.byref(ai), idx, 256, out, None, None, 0, None)

    assert call(kv_dtype=L.LSA_E4M3) == L.LSA_ERR_INVALID_ARG                       # scales missing
    assert call(kv_dtype=L.LSA_E4M3, k_scale=(3 << 20) + 2) == L.LSA_ERR_INVALID_ARG  # misaligned scales
    assert call(kv_dtype=L.LSA_E4M3, k_scale=3 << 20, k_row_stride=584, v_row_stride=584) == L.LSA_ERR_INVALID_ARG
    assert call(kv_dtype=7) == L.LSA_ERR_INVALID_ARG
    assert call(k_scale=3 << 20) == L.LSA_ERR_INVALID_ARG                            # scales on a bf16 cache
    small = L.AttnIn(1, 1, 8, 64, 64, 1024, 0.1, 16, 1 << 20, 2 << 20, 2 << 20, 64, 64, -1, -1, L.LSA_E4M3, 3 << 20)
    assert lib.lsa_sparse_attn(ctypes.byref(small), idx, 256, out, None, None, 0, None) == L.LSA_ERR_UNSUPPORTED


class _DeviceTensor:
    """Stands in for a CUDA tensor in the binding's argument checks (no GPU here)."""

    def __init__(self, shape, dtype, device=0, contiguous=True):
        import torch
        self.shape, self.dtype, self.is_cuda = torch.Size(shape), dtype, True
        self.device = torch.device("cuda", device)
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous

    def dim(self):
        return len(self.shape)

    def numel(self):
        return self.shape.numel()

    def element_size(self):
        import torch
        return torch.empty((), dtype=self.dtype).element_size()


def test_binding_checks_device_layout_dtype_and_shape(monkeypatch):
    import torch
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    i32 = torch.int32
    assert L._out(_DeviceTensor((2, 1, 2048), i32), "idx", i32, (2, 1, 2048)) is not None
    assert L._out(None, "idx", i32, (2, 1, 2048)) is None
    cases = [
        (torch.empty((2, 1, 2048), dtype=i32), "must be a CUDA tensor"),
        (_DeviceTensor((2, 1, 2048), i32, device=1), "current device"),
        (_DeviceTensor((2, 1, 2048), i32, contiguous=False), "contiguous"),
        (_DeviceTensor((2, 1, 2048), torch.int64), "dtype"),
        (_DeviceTensor((2, 2048), i32), "dims"),
        (_DeviceTensor((2, 1, 1024), i32), "shape"),   # a short idx would be written past its end
    ]
    for t, msg in cases:
        with pytest.raises(ValueError, match=msg):
            L._out(t, "idx", i32, (2, 1, 2048))
    with pytest.raises(ValueError, match="current device"):
        L._workspace(4096, None, _DeviceTensor((4096,), torch.uint8, device=1))
    with pytest.raises(ValueError, match="smaller"):
        L._workspace(4096, None, _DeviceTensor((4095,), torch.uint8))


def test_binding_checks_input_shapes_against_each_other(monkeypatch):
    import torch
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    q, k = _DeviceTensor((2, 1, 64, 128), bf), _DeviceTensor((2, 4096, 128), bf)
    w, sl = _DeviceTensor((2, 1, 64), f32), _DeviceTensor((2,), i32)
    for args, msg in [((q, w, _DeviceTensor((3, 4096, 128), bf), sl), "k has shape"),
                      ((q, w, _DeviceTensor((2, 4096, 64), bf), sl), "k has shape"),
                      ((q, _DeviceTensor((2, 1, 32), f32), k, sl), "w has shape"),
                      ((q, w, k, _DeviceTensor((1,), i32)), "seq_len has shape")]:
        with pytest.raises(ValueError, match=msg):
            L.indexer_in(*args)
    qa = _DeviceTensor((2, 1, 16, 64), bf)
    with pytest.raises(ValueError, match="v has shape"):
        L.attn_in(qa, sl, 0.125, k=_DeviceTensor((2, 4096, 64), bf), v=_DeviceTensor((2, 2048, 64), bf))
    with pytest.raises(ValueError, match="kv has shape"):
        L.attn_in(_DeviceTensor((2, 1, 128, 576), bf), sl, 0.04, kv=_DeviceTensor((1, 4096, 576), bf))
