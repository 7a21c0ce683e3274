"""ctypes binding of the LSA C ABI (include/lsa.h).

Argument marshalling only: every step of the path runs in the CUDA kernels of
liblsa.so. The functions carry the C names and take torch CUDA tensors; outputs
and workspaces are allocated with torch when the caller does not pass them.
There is no CPU fallback: if the library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblsa.so")

LSA_OK, LSA_ERR_INVALID_ARG, LSA_ERR_UNSUPPORTED, LSA_ERR_WORKSPACE, LSA_ERR_CUDA, LSA_ERR_TIMEOUT = range(6)
LSA_BF16, LSA_E4M3 = 0, 1
(LSA_OP_INDEX_FLAT, LSA_OP_INDEX_HIER, LSA_OP_SELECT, LSA_OP_SPARSE_ATTN, LSA_OP_LAYER_GROUP,
 LSA_OP_INDEX_COMPRESSED) = range(6)
LSA_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024   # static scratch of lsa_select_streaming_noalloc

EXPORTS = [
    "lsa_status_string", "lsa_last_error", "lsa_workspace_size", "lsa_index_flat", "lsa_select_streaming",
    "lsa_pool_pages", "lsa_index_hier", "lsa_sparse_attn", "lsa_layer_group", "lsa_device_status",
    "lsa_select_streaming_noalloc", "lsa_index_compressed", "lsa_pool_pages_e4m3", "lsa_index_hier_e4m3",
]


class LsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"[{status}] {msg}")
        self.status = status


class Budget(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int32), ("sink", ctypes.c_int32), ("window", ctypes.c_int32)]


class IndexerIn(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32),
                ("L_max", ctypes.c_int32), ("dtype", ctypes.c_int32), ("seq_len", ctypes.c_void_p),
                ("q", ctypes.c_void_p), ("q_scale", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("k", ctypes.c_void_p), ("k_scale", ctypes.c_void_p)]


class AttnIn(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("Hq", ctypes.c_int32), ("d_qk", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("L_max", ctypes.c_int32), ("scale", ctypes.c_float),
                ("seq_len", ctypes.c_void_p), ("q", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("k_row_stride", ctypes.c_int64), ("v_row_stride", ctypes.c_int64),
                ("stream_sink", ctypes.c_int32), ("stream_window", ctypes.c_int32),
                ("kv_dtype", ctypes.c_int32), ("k_scale", ctypes.c_void_p)]


class OpArgs(ctypes.Structure):
    _fields_ = [("indexer", ctypes.POINTER(IndexerIn)), ("attn", ctypes.POINTER(AttnIn)), ("budget", Budget),
                ("P", ctypes.c_int32), ("M", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("L_max", ctypes.c_int32),
                ("scores_external", ctypes.c_int32), ("m", ctypes.c_int32)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblsa.so (built by kv_indexing_b200.build). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m kv_indexing_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.lsa_status_string.restype = ctypes.c_char_p
    lib.lsa_status_string.argtypes = [i32]
    lib.lsa_last_error.restype = ctypes.c_char_p
    lib.lsa_last_error.argtypes = []
    lib.lsa_workspace_size.restype = i32
    lib.lsa_workspace_size.argtypes = [i32, ctypes.POINTER(OpArgs), ctypes.POINTER(sz)]
    lib.lsa_index_flat.restype = i32
    lib.lsa_index_flat.argtypes = [ctypes.POINTER(IndexerIn), Budget, vp, vp, vp, sz, vp]
    lib.lsa_index_compressed.restype = i32
    lib.lsa_index_compressed.argtypes = [ctypes.POINTER(IndexerIn), i32, Budget, vp, vp, vp, sz, vp]
    lib.lsa_select_streaming.restype = i32
    lib.lsa_select_streaming.argtypes = [vp, vp, i32, i32, i32, Budget, vp, vp, sz, vp]
    lib.lsa_select_streaming_noalloc.restype = i32
    lib.lsa_select_streaming_noalloc.argtypes = [vp, vp, i32, i32, i32, Budget, vp, vp]
    lib.lsa_pool_pages.restype = i32
    lib.lsa_pool_pages.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp]
    lib.lsa_pool_pages_e4m3.restype = i32
    lib.lsa_pool_pages_e4m3.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp]
    lib.lsa_index_hier_e4m3.restype = i32
    lib.lsa_index_hier_e4m3.argtypes = [ctypes.POINTER(IndexerIn), vp, vp, i32, i32, Budget, vp, vp, vp, sz, vp]
    lib.lsa_index_hier.restype = i32
    lib.lsa_index_hier.argtypes = [ctypes.POINTER(IndexerIn), vp, i32, i32, Budget, vp, vp, vp, sz, vp]
    lib.lsa_sparse_attn.restype = i32
    lib.lsa_sparse_attn.argtypes = [ctypes.POINTER(AttnIn), vp, i32, vp, vp, vp, sz, vp]
    lib.lsa_layer_group.restype = i32
    lib.lsa_layer_group.argtypes = [ctypes.POINTER(IndexerIn), vp, i32, i32, Budget, i32, ctypes.POINTER(AttnIn),
                                    ctypes.POINTER(vp), ctypes.POINTER(vp), vp, vp, sz, vp]
    lib.lsa_device_status.restype = i32
    lib.lsa_device_status.argtypes = [vp]
    _lib = lib
    return lib


def _check(st: int):
    if st != LSA_OK:
        lib = load()
        raise LsaError(st, f"{lib.lsa_status_string(st).decode()}: {lib.lsa_last_error().decode()}")


# ---------------------------------------------------------------------------
# torch marshalling helpers
# ---------------------------------------------------------------------------


def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return _torch().cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _need(t, name, dtype=None, dim=None):
    torch = _torch()
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    cur = torch.cuda.current_device()
    if t.device.index != cur:   # the kernels launch on the current device and would read another GPU's memory
        raise ValueError(f"{name} is on {t.device}, but the calls launch on the current device cuda:{cur}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None:
        dts = dtype if isinstance(dtype, tuple) else (dtype,)
        if t.dtype not in dts:
            raise ValueError(f"{name} has dtype {t.dtype}, expected {dts}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dims")
    return t


def _dims(t, name, shape):
    """t's shape must equal `shape` (None = any size in that place)."""
    if len(t.shape) != len(shape) or any(want is not None and got != want for got, want in zip(t.shape, shape)):
        want = tuple("*" if n is None else n for n in shape)
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want}")


def _out(t, name, dtype, shape):
    """A caller-supplied output (or None): a contiguous CUDA tensor on the current
    device with exactly the documented shape, since the kernels write all of it."""
    if t is None:
        return None
    _need(t, name, dtype, len(shape))
    _dims(t, name, shape)
    return t


def indexer_in(q, w, k, seq_len, q_scale=None, k_scale=None, m=1) -> IndexerIn:
    """Describe indexer tensors: q [B,T,H,d], w [B,T,H] f32, k [B,L_max,d], seq_len [B] i32.
    With m > 1, k holds one key per entry of m tokens: [B,L_max/m,d]."""
    torch = _torch()
    fp8 = q.dtype in (torch.float8_e4m3fn, torch.uint8)
    _need(q, "q", (torch.float8_e4m3fn, torch.uint8) if fp8 else torch.bfloat16, 4)
    _need(k, "k", (torch.float8_e4m3fn, torch.uint8) if fp8 else torch.bfloat16, 3)
    _need(w, "w", torch.float32, 3)
    _need(seq_len, "seq_len", torch.int32, 1)
    B, T, H, d = q.shape
    _dims(k, "k", (B, None, d))
    _dims(w, "w", (B, T, H))
    _dims(seq_len, "seq_len", (B,))
    if fp8:
        _need(q_scale, "q_scale", torch.float32, 3)
        _need(k_scale, "k_scale", torch.float32, 2)
        _dims(q_scale, "q_scale", (B, T, H))
        _dims(k_scale, "k_scale", (B, k.shape[1]))
    return IndexerIn(B, T, H, d, k.shape[1] * m, LSA_E4M3 if fp8 else LSA_BF16, _ptr(seq_len), _ptr(q),
                     _ptr(q_scale) if fp8 else None, _ptr(w), _ptr(k), _ptr(k_scale) if fp8 else None)


def attn_in(q, seq_len, scale, *, kv=None, k=None, v=None, d_v=None, stream_budget=None, kv_scale=None) -> AttnIn:
    """Describe attention tensors: q [B,T,Hq,d_qk]; MLA kv [B,L_max,d_qk] (V = first d_v
    columns) or separate k [B,L_max,d_qk], v [B,L_max,d_v]; all bf16, or an MLA kv of
    e4m3 codes (torch.float8_e4m3fn) with kv_scale [B,L_max] fp32 per token. stream_budget
    (k, sink, window) promises the index rows start with that streaming prefix."""
    torch = _torch()
    _need(q, "q", torch.bfloat16, 4)
    _need(seq_len, "seq_len", torch.int32, 1)
    B, T, Hq, d_qk = q.shape
    _dims(seq_len, "seq_len", (B,))
    ss, sw = (-1, -1) if stream_budget is None else (int(stream_budget[1]), int(stream_budget[2]))
    if kv is not None and kv.dtype == torch.float8_e4m3fn:
        _need(kv, "kv", torch.float8_e4m3fn, 3)
        _dims(kv, "kv", (B, None, None))
        if kv_scale is None:
            raise ValueError("an e4m3 kv needs kv_scale [B, L_max] float32")
        _need(kv_scale, "kv_scale", torch.float32, 2)
        if tuple(kv_scale.shape) != (kv.shape[0], kv.shape[1]):
            raise ValueError("kv_scale must be [B, L_max]")
        dv = d_v if d_v is not None else 512
        return AttnIn(B, T, Hq, d_qk, dv, kv.shape[1], float(scale), _ptr(seq_len), _ptr(q), _ptr(kv), _ptr(kv),
                      kv.shape[2], kv.shape[2], ss, sw, LSA_E4M3, _ptr(kv_scale))
    if kv_scale is not None:
        raise ValueError("kv_scale is for an e4m3 kv only")
    if kv is not None:
        _need(kv, "kv", torch.bfloat16, 3)
        _dims(kv, "kv", (B, None, None))
        dv = d_v if d_v is not None else (512 if d_qk == 576 else d_qk)
        return AttnIn(B, T, Hq, d_qk, dv, kv.shape[1], float(scale), _ptr(seq_len), _ptr(q), _ptr(kv), _ptr(kv),
                      kv.shape[2], kv.shape[2], ss, sw)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _dims(k, "k", (B, None, None))
    _dims(v, "v", (B, k.shape[1], None))
    return AttnIn(B, T, Hq, d_qk, v.shape[2], k.shape[1], float(scale), _ptr(seq_len), _ptr(q), _ptr(k), _ptr(v),
                  k.shape[2], v.shape[2], ss, sw)


def workspace_size(op: int, *, indexer: Optional[IndexerIn] = None, attn=None, budget=(1, 0, 0), P=0, M=0,
                   n_layers=0, B=0, T=0, L_max=0, scores_external=False, m=0) -> int:
    lib = load()
    a = OpArgs()
    keep = []
    if indexer is not None:
        a.indexer = ctypes.pointer(indexer)
    if attn is not None:
        if isinstance(attn, AttnIn):
            arr = (AttnIn * 1)(attn)
        else:
            arr = (AttnIn * len(attn))(*attn)
        keep.append(arr)
        a.attn = ctypes.cast(arr, ctypes.POINTER(AttnIn))
    a.budget = Budget(*budget)
    a.P, a.M, a.n_layers, a.B, a.T, a.L_max = P, M, n_layers, B, T, L_max
    a.scores_external = int(bool(scores_external))
    a.m = m
    out = ctypes.c_size_t(0)
    _check(lib.lsa_workspace_size(op, ctypes.byref(a), ctypes.byref(out)))
    return out.value


def _workspace(nbytes: int, device, workspace=None):
    torch = _torch()
    if nbytes == 0:
        return None
    if workspace is not None:
        _need(workspace, "workspace")
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace smaller than the {nbytes} bytes required")
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------


def lsa_index_flat(q, w, k, seq_len, budget, *, q_scale=None, k_scale=None, idx=None, scores_out=None,
                   with_idx=True, workspace=None, stream=None):
    """Flat indexing. Returns idx [B,T,k] int32 (or None when with_idx is False)."""
    torch = _torch()
    lib = load()
    ii = indexer_in(q, w, k, seq_len, q_scale, k_scale)
    B, T = q.shape[0], q.shape[1]
    if with_idx and idx is None:
        idx = torch.empty((B, T, budget[0]), dtype=torch.int32, device=q.device)
    if with_idx:
        _out(idx, "idx", torch.int32, (B, T, budget[0]))
    _out(scores_out, "scores_out", torch.float32, (B, T, k.shape[1]))
    need = workspace_size(LSA_OP_INDEX_FLAT, indexer=ii, budget=budget, scores_external=scores_out is not None)
    ws = _workspace(need, q.device, workspace)
    _check(lib.lsa_index_flat(ctypes.byref(ii), Budget(*budget), _ptr(idx) if with_idx else None, _ptr(scores_out),
                              _ptr(ws), _nbytes(ws), _stream(stream)))
    return idx if with_idx else None


def lsa_index_compressed(q, w, entry_keys, seq_len, m, budget, *, q_scale=None, k_scale=None, idx=None,
                         scores_out=None, with_idx=True, workspace=None, stream=None):
    """Indexing over compressed entries of m tokens: entry_keys [B,L_max/m,d]
    (seq_len in tokens; budget in entries). Returns idx [B,T,k] entry ids (or
    None when with_idx is False)."""
    torch = _torch()
    lib = load()
    ii = indexer_in(q, w, entry_keys, seq_len, q_scale, k_scale, m=m)
    B, T = q.shape[0], q.shape[1]
    if with_idx and idx is None:
        idx = torch.empty((B, T, budget[0]), dtype=torch.int32, device=q.device)
    if with_idx:
        _out(idx, "idx", torch.int32, (B, T, budget[0]))
    _out(scores_out, "scores_out", torch.float32, (B, T, entry_keys.shape[1]))
    need = workspace_size(LSA_OP_INDEX_COMPRESSED, indexer=ii, budget=budget, m=m,
                          scores_external=scores_out is not None)
    ws = _workspace(need, q.device, workspace)
    _check(lib.lsa_index_compressed(ctypes.byref(ii), m, Budget(*budget), _ptr(idx) if with_idx else None,
                                    _ptr(scores_out), _ptr(ws), _nbytes(ws), _stream(stream)))
    return idx if with_idx else None


def lsa_select_streaming(scores, seq_len, budget, *, idx=None, workspace=None, stream=None):
    """Streaming selection over given fp32 scores [B,T,L_max]. Returns idx [B,T,k]."""
    torch = _torch()
    lib = load()
    _need(scores, "scores", torch.float32, 3)
    _need(seq_len, "seq_len", torch.int32, 1)
    B, T, L_max = scores.shape
    _dims(seq_len, "seq_len", (B,))
    if idx is None:
        idx = torch.empty((B, T, budget[0]), dtype=torch.int32, device=scores.device)
    _out(idx, "idx", torch.int32, (B, T, budget[0]))
    need = workspace_size(LSA_OP_SELECT, budget=budget, B=B, T=T, L_max=L_max)
    ws = _workspace(need, scores.device, workspace)
    _check(lib.lsa_select_streaming(_ptr(scores), _ptr(seq_len), B, T, L_max, Budget(*budget), _ptr(idx), _ptr(ws),
                                    _nbytes(ws), _stream(stream)))
    return idx


def lsa_select_streaming_noalloc(scores, seq_len, budget, *, idx=None, stream=None):
    """lsa_select_streaming with the library's static scratch instead of a
    workspace: the C entry point allocates nothing, for callers that cannot
    allocate device memory where they select. Pass `idx` [B,T,k] int32 to keep
    this call free of allocations on the Python side too. Calls on one device
    share the scratch, so they must not overlap on the GPU."""
    torch = _torch()
    lib = load()
    _need(scores, "scores", torch.float32, 3)
    _need(seq_len, "seq_len", torch.int32, 1)
    B, T, L_max = scores.shape
    _dims(seq_len, "seq_len", (B,))
    if idx is None:
        idx = torch.empty((B, T, budget[0]), dtype=torch.int32, device=scores.device)
    _out(idx, "idx", torch.int32, (B, T, budget[0]))
    _check(lib.lsa_select_streaming_noalloc(_ptr(scores), _ptr(seq_len), B, T, L_max, Budget(*budget), _ptr(idx),
                                            _stream(stream)))
    return idx


def lsa_pool_pages(k, seq_len, P, *, page_keys=None, stream=None):
    """Mean-pooled page keys [B, L_max/P, d] bf16 from keys [B, L_max, d] bf16."""
    torch = _torch()
    lib = load()
    _need(k, "k", torch.bfloat16, 3)
    _need(seq_len, "seq_len", torch.int32, 1)
    B, L_max, d = k.shape
    _dims(seq_len, "seq_len", (B,))
    if page_keys is None:
        page_keys = torch.zeros((B, L_max // P, d), dtype=torch.bfloat16, device=k.device)
    _out(page_keys, "page_keys", torch.bfloat16, (B, L_max // P, d))
    _check(lib.lsa_pool_pages(_ptr(k), _ptr(seq_len), B, L_max, d, P, _ptr(page_keys), _stream(stream)))
    return page_keys


def lsa_index_hier(q, w, k, seq_len, page_keys, P, M, budget, *, idx=None, pages_out=None, workspace=None,
                   stream=None):
    """Hierarchical indexing. Returns (idx [B,T,k], pages [B,T,M] or None)."""
    torch = _torch()
    lib = load()
    ii = indexer_in(q, w, k, seq_len)
    _need(page_keys, "page_keys", torch.bfloat16, 3)
    if P > 0:
        _dims(page_keys, "page_keys", (q.shape[0], k.shape[1] // P, q.shape[3]))
    B, T = q.shape[0], q.shape[1]
    if idx is None:
        idx = torch.empty((B, T, budget[0]), dtype=torch.int32, device=q.device)
    _out(idx, "idx", torch.int32, (B, T, budget[0]))
    _out(pages_out, "pages_out", torch.int32, (B, T, M))
    need = workspace_size(LSA_OP_INDEX_HIER, indexer=ii, budget=budget, P=P, M=M)
    ws = _workspace(need, q.device, workspace)
    _check(lib.lsa_index_hier(ctypes.byref(ii), _ptr(page_keys), P, M, Budget(*budget), _ptr(idx), _ptr(pages_out),
                              _ptr(ws), _nbytes(ws), _stream(stream)))
    return idx, pages_out


def lsa_pool_pages_e4m3(k8, k_scale, seq_len, P, *, page_codes=None, page_scales=None, stream=None):
    """FP8 page keys from e4m3 token keys k8 [B, L_max, 128] with k_scale [B, L_max]:
    (page codes [B, L_max/P, 128] e4m3, page scales [B, L_max/P] fp32)."""
    torch = _torch()
    lib = load()
    _need(k8, "k8", (torch.float8_e4m3fn, torch.uint8), 3)
    _need(k_scale, "k_scale", torch.float32, 2)
    _need(seq_len, "seq_len", torch.int32, 1)
    B, L_max, d = k8.shape
    _dims(k_scale, "k_scale", (B, L_max))
    _dims(seq_len, "seq_len", (B,))
    if page_codes is None:
        page_codes = torch.zeros((B, L_max // P, d), dtype=torch.uint8, device=k8.device).view(k8.dtype)
    if page_scales is None:
        page_scales = torch.ones((B, L_max // P), dtype=torch.float32, device=k8.device)
    _out(page_codes, "page_codes", (torch.float8_e4m3fn, torch.uint8), (B, L_max // P, d))
    _out(page_scales, "page_scales", torch.float32, (B, L_max // P))
    _check(lib.lsa_pool_pages_e4m3(_ptr(k8), _ptr(k_scale), _ptr(seq_len), B, L_max, d, P, _ptr(page_codes),
                                   _ptr(page_scales), _stream(stream)))
    return page_codes, page_scales


def lsa_index_hier_e4m3(q8, q_scale, w, k8, k_scale, seq_len, page_codes, page_scales, P, M, budget, *, idx=None,
                        pages_out=None, workspace=None, stream=None):
    """FP8 hierarchical indexing. Returns (idx [B,T,k], pages [B,T,M] or None)."""
    torch = _torch()
    lib = load()
    ii = indexer_in(q8, w, k8, seq_len, q_scale, k_scale)
    _need(page_codes, "page_codes", (torch.float8_e4m3fn, torch.uint8), 3)
    _need(page_scales, "page_scales", torch.float32, 2)
    if P > 0:
        _dims(page_codes, "page_codes", (q8.shape[0], k8.shape[1] // P, q8.shape[3]))
        _dims(page_scales, "page_scales", (q8.shape[0], k8.shape[1] // P))
    B, T = q8.shape[0], q8.shape[1]
    if idx is None:
        idx = torch.empty((B, T, budget[0]), dtype=torch.int32, device=q8.device)
    _out(idx, "idx", torch.int32, (B, T, budget[0]))
    _out(pages_out, "pages_out", torch.int32, (B, T, M))
    need = workspace_size(LSA_OP_INDEX_HIER, indexer=ii, budget=budget, P=P, M=M)
    ws = _workspace(need, q8.device, workspace)
    _check(lib.lsa_index_hier_e4m3(ctypes.byref(ii), _ptr(page_codes), _ptr(page_scales), P, M, Budget(*budget),
                                   _ptr(idx), _ptr(pages_out), _ptr(ws), _nbytes(ws), _stream(stream)))
    return idx, pages_out


def lsa_sparse_attn(q, idx, seq_len, scale, *, kv=None, k=None, v=None, d_v=None, out=None, lse=None,
                    workspace=None, stream=None, stream_budget=None, kv_scale=None):
    """Sparse attention over idx [B,T,k]. Returns (out [B,T,Hq,d_v] bf16, lse or None).
    stream_budget (k, sink, window): idx rows come from the streaming selection with
    that budget, so their sink/window prefix may be computed instead of read.
    An e4m3 MLA kv (torch.float8_e4m3fn) takes kv_scale [B, L_max] fp32."""
    torch = _torch()
    lib = load()
    ai = attn_in(q, seq_len, scale, kv=kv, k=k, v=v, d_v=d_v, stream_budget=stream_budget, kv_scale=kv_scale)
    _need(idx, "idx", torch.int32, 3)
    if tuple(idx.shape[:2]) != (ai.B, ai.T):
        raise ValueError(f"idx has shape {tuple(idx.shape)}, expected [{ai.B}, {ai.T}, k]")
    if out is None:
        out = torch.empty((ai.B, ai.T, ai.Hq, ai.d_v), dtype=torch.bfloat16, device=q.device)
    _out(out, "out", torch.bfloat16, (ai.B, ai.T, ai.Hq, ai.d_v))
    _out(lse, "lse", torch.float32, (ai.B, ai.T, ai.Hq))
    need = workspace_size(LSA_OP_SPARSE_ATTN, attn=ai, budget=(idx.shape[2], 0, 0))
    ws = _workspace(need, q.device, workspace)
    _check(lib.lsa_sparse_attn(ctypes.byref(ai), _ptr(idx), idx.shape[2], _ptr(out), _ptr(lse), _ptr(ws), _nbytes(ws),
                               _stream(stream)))
    return out, lse


def lsa_layer_group(q, w, k, seq_len, budget, layers: Sequence[dict], *, P=0, M=0, page_keys=None, outs=None,
                    lses=None, idx=None, workspace=None, stream=None):
    """One indexing pass (flat if P == 0) feeding len(layers) sparse-attention layers.

    Each layer dict: q, scale and kv (MLA) or k/v. Returns (idx, outs)."""
    torch = _torch()
    lib = load()
    ii = indexer_in(q, w, k, seq_len)
    ais = [attn_in(l["q"], seq_len, l["scale"], kv=l.get("kv"), k=l.get("k"), v=l.get("v"), d_v=l.get("d_v"),
                   kv_scale=l.get("kv_scale"))
           for l in layers]
    n = len(ais)
    if outs is None:
        outs = [torch.empty((a.B, a.T, a.Hq, a.d_v), dtype=torch.bfloat16, device=q.device) for a in ais]
    if idx is None:
        idx = torch.empty((q.shape[0], q.shape[1], budget[0]), dtype=torch.int32, device=q.device)
    _out(idx, "idx", torch.int32, (q.shape[0], q.shape[1], budget[0]))
    if len(outs) != n or (lses is not None and len(lses) != n):
        raise ValueError(f"outs and lses need one entry per layer ({n})")
    for i, a in enumerate(ais):
        _out(outs[i], f"outs[{i}]", torch.bfloat16, (a.B, a.T, a.Hq, a.d_v))
        if lses is not None:
            _out(lses[i], f"lses[{i}]", torch.float32, (a.B, a.T, a.Hq))
    if page_keys is not None:
        _out(page_keys, "page_keys", torch.bfloat16, (q.shape[0], k.shape[1] // P if P else 0, k.shape[2]))
    need = workspace_size(LSA_OP_LAYER_GROUP, indexer=ii, attn=ais, budget=budget, P=P, M=M, n_layers=n)
    ws = _workspace(need, q.device, workspace)
    arr = (AttnIn * n)(*ais)
    outp = (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs])
    lsep = (ctypes.c_void_p * n)(*[(_ptr(l) if l is not None else None) for l in (lses or [None] * n)])
    _check(lib.lsa_layer_group(ctypes.byref(ii), _ptr(page_keys), P, M, Budget(*budget), n, arr, outp, lsep,
                               _ptr(idx), _ptr(ws), _nbytes(ws), _stream(stream)))
    return idx, outs


def lsa_device_status(stream=None) -> int:
    """Synchronise and return the device status word (0 = ok); raises on timeout."""
    lib = load()
    st = lib.lsa_device_status(_stream(stream))
    _check(st)
    return st
