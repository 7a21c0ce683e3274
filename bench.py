#!/usr/bin/env python
"""Benchmark of the LSA hot path on B200.

One step = one pass of the whole path over one batch: lightning-indexer scores
(tcgen05) -> streaming top-k -> sparse MLA attention (+ split combine). The
default workload is flat decode (8 sequences x 131072 cached tokens, one query
each, top-k 2048 = sink 64 + window 960 + 1024 dynamic; 128 query heads,
d_qk 576 / d_v 512). Inputs are seeded synthetic data resident in HBM; L2 is
flushed (256 MiB write) between timed steps, outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--fp8] [--fp8-kv]

Workloads (kv_indexing_b200.inputs.WORKLOADS): flat_decode_128k (default),
flat_decode_1m and hier_decode_1m (the same 2 x 1M inputs, hierarchy off / on;
page pooling timed once, outside the step), cli_group_256k(_flat) (one indexing
pass feeding two layers), prefill_64k (4096 causal queries; --fp8 for e4m3
indexer inputs), compressed_decode_1m (262144 entries of 4 tokens; --fp8 for
e4m3 entry keys), and hier_sweep: flat against hierarchical indexing on the
same inputs at L = 64K, 256K, 512K and 1M (B=2). --fp8-kv stores every
workload's latent attention cache as e4m3 codes with a per-token fp32 scale.

Each line carries: the device-timed step (one CUDA graph per step, no events
inside) and its per-stage breakdown (a second graph with events between the
stages), the same step as plain stream launches, the roofline of the dominant
kernel, `e2e` (the public API with the step's queries copied in from pinned
host memory and o, idx copied out, split into copy, compute and host-issue
time; also with the user's calls captured in a CUDA graph), and `cpu_baseline`
(the C++ oracle on the host cores: all cores over the rows, and one thread).

Prints one JSON line (rank 0). Under torchrun each rank runs its own batch
(weak scaling, no data-path collective); times are device times, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode queries/s (indexer+top-k+sparse attn) at 128K-1M; % of HBM/TC roofline"
UNIT = "queries/s"
SWEEP_L = (65536, 262144, 524288, 1048576)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    from kv_indexing_b200.inputs import WORKLOADS
    p.add_argument("--workload", default="flat_decode_128k", choices=sorted(WORKLOADS) + ["hier_sweep"])
    p.add_argument("--seed", type=int, default=1)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--fp8", action="store_true", help="e4m3 indexer keys and queries (prefill, compressed)")
    p.add_argument("--fp8-kv", action="store_true",
                   help="e4m3 latent KV cache (per-token scale) for the sparse MLA attention")
    return p.parse_args()


# ---------------------------------------------------------------------------
# algorithmic work per query (what the method must move), used for the roofline
# ---------------------------------------------------------------------------


def indexer_bytes_per_query(w, fp8=False, n_keys=None) -> int:
    """Keys streamed once (+ their e4m3 scales) + the query's vectors and head weights."""
    n = w.L if n_keys is None else n_keys
    if fp8:
        return n * w.d + n * 4 + w.H * w.d + w.H * 4 + w.H * 4
    return n * w.d * 2 + w.H * w.d * 2 + w.H * 4


def hier_index_bytes_per_query(w, fp8=False) -> int:
    """Page keys of the whole sequence + the recalled pages' token keys + q, w
    (e4m3: one byte per element plus a 4-byte scale per page, token and query head)."""
    if fp8:
        return ((w.L // w.P) * (w.d + 4) + w.M * w.P * (w.d + 4) + w.H * (w.d + 4) + w.H * 4)
    return (w.L // w.P) * w.d * 2 + w.M * w.P * w.d * 2 + w.H * w.d * 2 + w.H * 4


def attention_bytes_per_query(w, kv8=False) -> int:
    """Gathered latent KV rows (e4m3: codes + a 4-byte scale per row) + q + o."""
    row = w.d_qk + 4 if kv8 else w.d_qk * 2
    return w.k * row + w.Hq * w.d_qk * 2 + w.Hq * w.d_v * 2


def prefill_indexer_flops(w) -> float:
    """2 H d per visible (query, key) pair, causal."""
    return 2.0 * w.H * w.d * sum(p + 1 for p in range(w.L - w.T, w.L)) * w.B


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_traffic(name: str):
    """DRAM bytes per launch from a committed ncu capture, or None when the kernel
    source changed since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            tab = json.load(f)
    except OSError:
        return None
    ent = tab.get(name)
    if not ent:
        return None
    try:
        sha = hashlib.sha256(open(os.path.join(ROOT, ent["source_file"]), "rb").read()).hexdigest()
    except OSError:
        return None
    return ent["dram_bytes_per_launch"] if sha == ent["source_sha256"] else None


# ---------------------------------------------------------------------------
# multi-rank plumbing (one process per GPU; weak scaling, no data-path collective)
# ---------------------------------------------------------------------------


def rank_seed(seed: int, rank: int) -> int:
    """Each rank times its own independent batch."""
    return seed + 1000 * rank


def max_over_ranks(x: float, dev, pg) -> float:
    """Whole-job time = the slowest rank's device time."""
    if not pg:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------


class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, uuid: str, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop = period_s, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            u = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(u)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.reason_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            self.nv = None
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.reason_fn(self.h)
                for k, bit in self.REASONS.items():
                    if mask & bit and k != "gpu_idle":
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def workload_config(w, **extra):
    c = {"workload": w.name, "B": w.B, "L": w.L, "T": w.T, "H_I": w.H, "d_I": w.d, "k": w.k, "sink": w.sink,
         "window": w.window, "Hq": w.Hq, "d_qk": w.d_qk, "d_v": w.d_v, "P": w.P, "M": w.M,
         "n_layers": w.n_layers, "entry_tokens_m": w.m,
         "l2": "flushed between timed steps (256 MiB write, outside the timed events)"}
    c.update(extra)
    return c


def kind_of(w) -> str:
    if w.m:
        return "compressed"
    if w.n_layers > 1:
        return "group"
    if w.P:
        return "hier"
    return "prefill" if w.T > 1 else "flat"


def host_inputs(w, seed, fp8=False):
    """Indexer inputs from the seeded host generator (needles included); for
    compressed entries the entry keys take the place of the token keys. With
    fp8, e4m3 codes and row scales are drawn too."""
    from kv_indexing_b200 import inputs as I
    if fp8 and not w.fp8:
        w = I.scaled(w, fp8=True)
    if w.m:
        x = I.make_compressed_inputs(w, seed)
        x["k_idx"] = x.pop("entry_keys")
        if "entry_keys_fp8" in x:
            x["k_idx_fp8"] = x.pop("entry_keys_fp8")
        return x
    return I.make_indexer_inputs(w, seed)


# ---------------------------------------------------------------------------
# the path of one workload on the device: stages of a step, the public-API
# step a user calls, and what the roofline measures
# ---------------------------------------------------------------------------


class Path:
    def __init__(self, torch, L, w, x, dev, seed, fp8, layers=None, kv8=False):
        import numpy as np
        self.torch, self.L, self.w, self.x, self.dev, self.fp8, self.kv8 = torch, L, w, x, dev, fp8, kv8
        self.kind = kind_of(w)
        B, T = w.B, w.T
        self.budget = (w.k, w.sink, w.window)

        def up(arr, kind):
            t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16) if kind == "bf16" else
                                 np.ascontiguousarray(arr))
            t = t.view(torch.bfloat16) if kind == "bf16" else t
            return t.to(dev)

        self.up = up
        self.q, self.k, self.wt, self.sl = up(x["q_idx"], "bf16"), up(x["k_idx"], "bf16"), up(x["w"], "f32"), \
            up(x["seq_len"], "i32")
        self.qs = self.ks = None
        if fp8:
            if "k_idx_fp8" not in x:
                raise SystemExit(f"workload {w.name} has no e4m3 indexer inputs")
            self.q = up(x["q_idx_fp8"], "u8").view(torch.float8_e4m3fn)
            self.k = up(x["k_idx_fp8"], "u8").view(torch.float8_e4m3fn)
            self.qs, self.ks = up(x["q_scale"], "f32"), up(x["k_scale"], "f32")
        kv_rows = w.L // w.m if w.m else w.L
        self.layers = layers if layers is not None else []
        for li in range(0 if layers is not None else w.n_layers):
            qa = device_bf16_normal(torch, (B, T, w.Hq, w.d_qk), 7919 * seed + 2 * li, dev)
            kv = device_bf16_normal(torch, (B, kv_rows, w.d_qk), 7919 * seed + 2 * li + 1, dev)
            lay = {"q": qa, "kv": kv, "scale": w.scale, "d_v": w.d_v}
            if kv8:   # per-token e4m3: scale = amax / 448, codes = kv / scale (round to nearest even)
                kf = kv.float()
                amax = kf.abs().amax(dim=-1)
                sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).contiguous()
                lay["kv"] = (kf / sc[..., None]).to(torch.float8_e4m3fn).contiguous()
                lay["kv_scale"] = sc
                del kf
            self.layers.append(lay)
        self.idx = torch.empty((B, T, w.k), dtype=torch.int32, device=dev)
        self.outs = [torch.empty((B, T, w.Hq, w.d_v), dtype=torch.bfloat16, device=dev) for _ in range(w.n_layers)]
        self.extra = {}
        self.breakdown_stages = None
        self._build()

    def _ws(self, n):
        return self.torch.empty(max(256, n), dtype=self.torch.uint8, device=self.dev)

    def _build(self):
        torch, L, w = self.torch, self.L, self.w
        B, T, budget = w.B, w.T, self.budget
        q, k, wt, sl, qs, ks = self.q, self.k, self.wt, self.sl, self.qs, self.ks
        lay0 = self.layers[0]
        # attention rows: entries for compressed indexing (decode: the query's entry
        # position is seq_len // m - 1), tokens otherwise
        self.sl_attn = torch.div(sl, w.m, rounding_mode="floor").to(torch.int32) if w.m else sl
        ai = L.attn_in(lay0["q"], self.sl_attn, w.scale, kv=lay0["kv"], d_v=w.d_v, stream_budget=budget,
                       kv_scale=lay0.get("kv_scale"))
        self.attn_ws = self._ws(L.workspace_size(L.LSA_OP_SPARSE_ATTN, attn=ai, budget=(w.k, 0, 0)))

        def attn(li, idx=None):
            lay = self.layers[li]
            return lambda s: L.lsa_sparse_attn(lay["q"], self.idx if idx is None else idx, self.sl_attn, w.scale,
                                               kv=lay["kv"], d_v=w.d_v, out=self.outs[li], workspace=self.attn_ws,
                                               stream_budget=budget, stream=s, kv_scale=lay.get("kv_scale"))

        kind = self.kind
        if kind in ("flat", "prefill", "compressed"):
            n_slots = w.L // w.m if w.m else w.L
            self.scores = torch.empty((B, T, n_slots), dtype=torch.float32, device=self.dev)
            sl_sel = self.sl_attn
            self.sel_ws = self._ws(L.workspace_size(L.LSA_OP_SELECT, budget=budget, B=B, T=T, L_max=n_slots))
            if w.m:
                ii = L.indexer_in(q, wt, k, sl, qs, ks, m=w.m)
                self.api_ws = self._ws(L.workspace_size(L.LSA_OP_INDEX_COMPRESSED, indexer=ii, budget=budget, m=w.m))
                index_scores = lambda s: L.lsa_index_compressed(q, wt, k, sl, w.m, budget, q_scale=qs, k_scale=ks,
                                                                 scores_out=self.scores, with_idx=False, stream=s)
            else:
                ii = L.indexer_in(q, wt, k, sl, qs, ks)
                self.api_ws = self._ws(L.workspace_size(L.LSA_OP_INDEX_FLAT, indexer=ii, budget=budget))
                index_scores = lambda s: L.lsa_index_flat(q, wt, k, sl, budget, q_scale=qs, k_scale=ks,
                                                          scores_out=self.scores, with_idx=False, stream=s)
            if w.m:
                index_call = lambda s: L.lsa_index_compressed(q, wt, k, sl, w.m, budget, q_scale=qs, k_scale=ks,
                                                              idx=self.idx, workspace=self.api_ws, stream=s)
            else:
                index_call = lambda s: L.lsa_index_flat(q, wt, k, sl, budget, q_scale=qs, k_scale=ks, idx=self.idx,
                                                        workspace=self.api_ws, stream=s)
            # the step: the indexing call (scores and selection, fused where the
            # selection uses the indexer's summaries) then attention; the
            # breakdown splits the indexing call into scores alone and selection
            self.stages = [("index", index_call), ("attention", attn(0))]
            self.breakdown_stages = [("indexer", index_scores),
                                     ("select", lambda s: L.lsa_select_streaming(self.scores, sl_sel, budget,
                                                                                 idx=self.idx, workspace=self.sel_ws,
                                                                                 stream=s)),
                                     ("attention", attn(0))]
            self.dominant = "indexer"
            if kind == "prefill":
                self.roof_kernel = "indexer (tcgen05 score GEMM over causal tiles, fused epilogue)"
                self.roof_flops = prefill_indexer_flops(w)
            else:
                n_keys = w.L // w.m if w.m else w.L
                self.roof_kernel = ("entry " if w.m else "") + "indexer (tcgen05 score GEMM + fused epilogue)"
                self.roof_bytes = indexer_bytes_per_query(w, self.fp8, n_keys) * B * T
        elif kind == "hier":
            self._pool_once()
            ii = L.indexer_in(q, wt, k, sl, qs, ks)
            self.api_ws = self._ws(L.workspace_size(L.LSA_OP_INDEX_HIER, indexer=ii, budget=budget, P=w.P, M=w.M))
            if self.fp8:
                hier_call = lambda s: L.lsa_index_hier_e4m3(q, qs, wt, k, ks, sl, self.page_keys, self.page_scales,
                                                            w.P, w.M, budget, idx=self.idx, workspace=self.api_ws,
                                                            stream=s)
            else:
                hier_call = lambda s: L.lsa_index_hier(q, wt, k, sl, self.page_keys, w.P, w.M, budget, idx=self.idx,
                                                       workspace=self.api_ws, stream=s)
            self.stages = [("hier_index", hier_call), ("attention", attn(0))]
            self.dominant = "hier_index"
            self.roof_kernel = "hierarchical indexing call (page scores, page recall, fine scores, token top-k)"
            self.roof_bytes = hier_index_bytes_per_query(w, self.fp8) * B * T
        else:   # group
            if w.P:
                self._pool_once()
            ii = L.indexer_in(q, wt, k, sl)
            ais = [L.attn_in(l["q"], sl, w.scale, kv=l["kv"], d_v=w.d_v, kv_scale=l.get("kv_scale")) for l in self.layers]
            self.api_ws = self._ws(L.workspace_size(L.LSA_OP_LAYER_GROUP, indexer=ii, attn=ais, budget=budget,
                                                    P=w.P, M=w.M, n_layers=w.n_layers))
            pk = self.page_keys if w.P else None
            self.stages = [("group", lambda s: L.lsa_layer_group(q, wt, k, sl, budget, self.layers, P=w.P, M=w.M,
                                                                 page_keys=pk, outs=self.outs, idx=self.idx,
                                                                 workspace=self.api_ws, stream=s))]
            # the indexing pass alone (timed beside the step: its cost over the N layers
            # is the per-layer amortised indexer cost)
            self.idx_only = torch.empty_like(self.idx)
            if w.P:
                hws = self._ws(L.workspace_size(L.LSA_OP_INDEX_HIER, indexer=ii, budget=budget, P=w.P, M=w.M))
                self.index_alone = [("index_alone", lambda s: L.lsa_index_hier(
                    q, wt, k, sl, pk, w.P, w.M, budget, idx=self.idx_only, workspace=hws, stream=s))]
            else:
                fws = self._ws(L.workspace_size(L.LSA_OP_INDEX_FLAT, indexer=ii, budget=budget))
                self.index_alone = [("index_alone", lambda s: L.lsa_index_flat(
                    q, wt, k, sl, budget, idx=self.idx_only, workspace=fws, stream=s))]
            self.dominant = "group"
            self.roof_kernel = f"layer-group call (one indexing pass + {w.n_layers} attention layers)"
            ib = hier_index_bytes_per_query(w) if w.P else indexer_bytes_per_query(w)
            self.roof_bytes = (ib + w.n_layers * attention_bytes_per_query(w, self.kv8)) * B * T

    def _pool_once(self):
        torch, L, w = self.torch, self.L, self.w
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if self.fp8:
            self.page_keys = torch.zeros((w.B, w.L // w.P, w.d), dtype=torch.uint8,
                                         device=self.dev).view(torch.float8_e4m3fn)
            self.page_scales = torch.ones((w.B, w.L // w.P), dtype=torch.float32, device=self.dev)
            e0.record()
            L.lsa_pool_pages_e4m3(self.k, self.ks, self.sl, w.P, page_codes=self.page_keys,
                                  page_scales=self.page_scales)
            e1.record()
        else:
            self.page_keys = torch.zeros((w.B, w.L // w.P, w.d), dtype=torch.bfloat16, device=self.dev)
            e0.record()
            L.lsa_pool_pages(self.k, self.sl, w.P, page_keys=self.page_keys)
            e1.record()
        torch.cuda.synchronize()
        self.extra["page_pooling_once_us"] = 1000 * e0.elapsed_time(e1)

    # -- the public-API step a user calls, on given device inputs ------------
    def api_index(self, s, q, wt):
        """The indexing call of the step (not for the layer group)."""
        L, w, budget = self.L, self.w, self.budget
        k, sl, qs, ks = self.k, self.sl, self.qs, self.ks
        if self.kind == "hier" and self.fp8:
            L.lsa_index_hier_e4m3(q, qs, wt, k, ks, sl, self.page_keys, self.page_scales, w.P, w.M, budget,
                                  idx=self.idx, workspace=self.api_ws, stream=s)
        elif self.kind == "hier":
            L.lsa_index_hier(q, wt, k, sl, self.page_keys, w.P, w.M, budget, idx=self.idx, workspace=self.api_ws,
                             stream=s)
        elif self.kind == "compressed":
            L.lsa_index_compressed(q, wt, k, sl, w.m, budget, q_scale=qs, k_scale=ks, idx=self.idx,
                                   workspace=self.api_ws, stream=s)
        else:
            L.lsa_index_flat(q, wt, k, sl, budget, q_scale=qs, k_scale=ks, idx=self.idx, workspace=self.api_ws,
                             stream=s)

    def api_attend(self, s, qas):
        """The attention call of the step over self.idx (not for the layer group)."""
        lay = self.layers[0]
        self.L.lsa_sparse_attn(qas[0], self.idx, self.sl_attn, self.w.scale, kv=lay["kv"], d_v=self.w.d_v,
                               out=self.outs[0], workspace=self.attn_ws, stream_budget=self.budget, stream=s,
                               kv_scale=lay.get("kv_scale"))

    def api_step(self, s, q, wt, qas):
        """The path through the library's public calls (what an application
        issues per decode step), reading the queries from q, wt and qas."""
        L, w, budget = self.L, self.w, self.budget
        k, sl, qs, ks = self.k, self.sl, self.qs, self.ks
        if self.kind == "group":
            layers = [dict(l, q=qa) for l, qa in zip(self.layers, qas)]
            L.lsa_layer_group(q, wt, k, sl, budget, layers, P=w.P, M=w.M,
                              page_keys=self.page_keys if w.P else None, outs=self.outs, idx=self.idx,
                              workspace=self.api_ws, stream=s)
            return
        self.api_index(s, q, wt)
        self.api_attend(s, qas)


def device_bf16_normal(torch, shape, seed, dev):
    """Seeded N(0,1) bf16 drawn on the device (latent KV caches and attention
    queries; the long caches would take minutes on the host generator)."""
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    flat = out.view(-1)
    step = 1 << 28
    for lo in range(0, flat.numel(), step):          # bounded float32 temporaries
        n = min(step, flat.numel() - lo)
        flat[lo:lo + n] = torch.randn((n,), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    return out


# ---------------------------------------------------------------------------
# device timing
# ---------------------------------------------------------------------------


def capture(torch, stages, dev, stream, inner_events, keep_graph=False):
    n = len(stages)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n + 1)]
    g = torch.cuda.CUDAGraph(keep_graph=keep_graph)
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
        s = torch.cuda.current_stream(dev)
        ev[0].record(s)
        for i, (_, fn) in enumerate(stages):
            fn(s)
            if inner_events or i == n - 1:
                ev[i + 1].record(s)
    torch.cuda.synchronize()
    launches = None
    if keep_graph:
        launches = graph_kernel_count(g)
        g.instantiate()
    return g, ev, launches


def graph_kernel_count(g):
    """Kernel nodes of a captured graph (our launches per step), or None."""
    try:
        from cuda.bindings import runtime as rt
    except Exception:
        try:
            from cuda import cudart as rt
        except Exception:
            return None
    try:
        raw = g.raw_cuda_graph()
        graph = rt.cudaGraph_t(init_value=raw) if hasattr(rt, "cudaGraph_t") else raw
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes]
        return sum(1 for t in kinds if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:
        return None


def time_device(torch, stages, K, warmup, flush, dev, pg, breakdown_stages=None):
    """Whole step as one graph (events only around it), per-stage breakdown from
    a second graph (of breakdown_stages when given: the same work split into
    finer calls), and the same step as plain launches. Returns a dict."""
    import torch.distributed as dist
    stream = torch.cuda.current_stream(dev)
    bstages = breakdown_stages or stages
    for _ in range(max(3, warmup)):
        flush()
        for _, fn in stages:
            fn(stream)
        flush()
        for _, fn in bstages:
            fn(stream)
    torch.cuda.synchronize()
    g, ev, launches = capture(torch, stages, dev, stream, inner_events=False, keep_graph=True)
    gb, evb, _ = capture(torch, bstages, dev, stream, inner_events=True)
    n = len(stages)
    nb = len(bstages)
    for _ in range(3):
        flush()
        g.replay()
        flush()
        gb.replay()
    torch.cuda.synchronize()
    step = []
    if pg:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        for _ in range(K):
            flush()
            g.replay()
            torch.cuda.synchronize()
            step.append(ev[0].elapsed_time(ev[n]))
    torch.cuda.synchronize()
    if pg:
        dist.barrier()
    per = [[] for _ in range(nb)]
    for _ in range(K):
        flush()
        gb.replay()
        torch.cuda.synchronize()
        for i in range(nb):
            per[i].append(evb[i].elapsed_time(evb[i + 1]))
    # plain launches: the same calls issued on the stream, no graph
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    plain = []
    for _ in range(K):
        flush()
        e0.record(stream)
        for _, fn in stages:
            fn(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        plain.append(e0.elapsed_time(e1))
    del g, gb
    return {
        "ms_per_step": max_over_ranks(float(sum(step)) / K, dev, pg),
        "step_ms_median": statistics.median(step),
        "breakdown_us": {name: 1000 * sum(per[i]) / K for i, (name, _) in enumerate(bstages)},
        "plain_ms_per_step": max_over_ranks(float(sum(plain)) / K, dev, pg),
        "clocks": clk.summary(),
        "launches_per_step": launches,
    }


def time_e2e(torch, path, K, flush, dev, pg):
    """End to end through the public API: per step the step's queries go in
    from pinned host memory (indexer q [+ q scales], head weights, attention q of
    every layer) and o of every layer and idx come back, timed with events on
    the stream. Three ways an application issues the same public calls:
      plain      copies in, the calls, copies out, one after another on a stream
                 (split into copy, compute and host-issue time);
      overlap    the attention queries (most of the bytes in) cross on a second
                 stream while the indexing call runs, idx comes back while the
                 attention runs; o comes back last;
      graph      the overlapped sequence captured once in a CUDA graph and
                 replayed per step (what a serving loop does; no host issue cost).
    The line's e2e value is the graph one."""
    stream = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)
    qi_srcs = [path.q, path.wt] + ([path.qs] if path.qs is not None else [])   # the indexing call's queries
    qa_srcs = [l["q"] for l in path.layers]                                   # the attention queries
    h_qi = [t.cpu().pin_memory() for t in qi_srcs]
    h_qa = [t.cpu().pin_memory() for t in qa_srcs]
    d_qi = [torch.empty_like(t) for t in qi_srcs]
    d_qa = [torch.empty_like(t) for t in qa_srcs]
    h_o = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in path.outs]
    h_idx = torch.empty(path.idx.shape, dtype=path.idx.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in h_qi + h_qa)
    d2h = sum(t.numel() * t.element_size() for t in h_o) + h_idx.numel() * h_idx.element_size()
    grouped = path.kind == "group"

    def with_queries(fn):
        qs_saved = path.qs
        if path.qs is not None:
            path.qs = d_qi[2]
        try:
            fn()
        finally:
            path.qs = qs_saved

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    def plain():
        ev[0].record(stream)
        for d, h in zip(d_qi + d_qa, h_qi + h_qa):
            d.copy_(h, non_blocking=True)
        ev[1].record(stream)
        t0 = time.perf_counter()
        with_queries(lambda: path.api_step(stream, d_qi[0], d_qi[1], d_qa))
        host = time.perf_counter() - t0
        ev[2].record(stream)
        for h, d in zip(h_o + [h_idx], path.outs + [path.idx]):
            h.copy_(d, non_blocking=True)
        ev[3].record(stream)
        return host

    e_start, e_qa, e_idx, e_side = (torch.cuda.Event() for _ in range(4))

    def overlap(s):
        # s: the main stream (the capture stream inside a graph). A copy engine
        # serves copies in the order they are issued, so the indexing call's
        # small queries go first and the attention queries fork off after them.
        with torch.cuda.stream(s):
            for d, h in zip(d_qi, h_qi):
                d.copy_(h, non_blocking=True)
        e_start.record(s)
        side.wait_event(e_start)
        with torch.cuda.stream(side):
            for d, h in zip(d_qa, h_qa):
                d.copy_(h, non_blocking=True)
        e_qa.record(side)
        if grouped:
            s.wait_event(e_qa)
            with_queries(lambda: path.api_step(s, d_qi[0], d_qi[1], d_qa))
        else:
            with_queries(lambda: path.api_index(s, d_qi[0], d_qi[1]))
            e_idx.record(s)
            side.wait_event(e_idx)
            with torch.cuda.stream(side):
                h_idx.copy_(path.idx, non_blocking=True)
            s.wait_event(e_qa)
            path.api_attend(s, d_qa)
        e_side.record(side)
        with torch.cuda.stream(s):
            for h, d in zip(h_o, path.outs):
                h.copy_(d, non_blocking=True)
            if grouped:
                h_idx.copy_(path.idx, non_blocking=True)
        s.wait_event(e_side)

    def timed(fn):
        flush()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        r = fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1), r

    for _ in range(3):
        timed(plain)
    rec = []
    for _ in range(K):
        flush()
        torch.cuda.synchronize()
        host = plain()
        torch.cuda.synchronize()
        rec.append((ev[0].elapsed_time(ev[3]), ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]),
                    ev[2].elapsed_time(ev[3]), 1000 * host))
    for _ in range(3):
        timed(lambda: overlap(stream))
    rec_o = [timed(lambda: overlap(stream))[0] for _ in range(K)]
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
        overlap(torch.cuda.current_stream(dev))
    torch.cuda.synchronize()
    for _ in range(3):
        timed(g.replay)
    rec_g = [timed(g.replay)[0] for _ in range(K)]
    del g
    units = path.w.B * path.w.T * (int(os.environ.get("WORLD_SIZE", "1")))
    mean = lambda rs, i: sum(r[i] for r in rs) / K
    tp = max_over_ranks(mean(rec, 0), dev, pg)
    to = max_over_ranks(sum(rec_o) / K, dev, pg)
    tg = max_over_ranks(sum(rec_g) / K, dev, pg)
    return {
        "value": units / (tg / 1000.0), "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
        "ms_per_step": tg, "mode": "graph (the overlapped calls captured once, replayed per step)",
        "overlap": {"value": units / (to / 1000.0), "ms_per_step": to},
        "plain": {"value": units / (tp / 1000.0), "ms_per_step": tp, "h2d_ms": mean(rec, 1),
                  "compute_ms": mean(rec, 2), "d2h_ms": mean(rec, 3), "host_issue_ms": mean(rec, 4)},
        "note": "caches resident; per step the new queries go in and o, idx come out (pinned host memory)",
    }


# ---------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------


def host_bf16(t):
    import numpy as np
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_layer(lay):
    """A device layer's query and cache as the oracle takes them (e4m3 codes and scales, or bf16)."""
    import numpy as np
    import torch
    if "kv_scale" in lay:
        return {"qa": host_bf16(lay["q"]), "kv8": lay["kv"].view(torch.uint8).cpu().numpy(),
                "ks": lay["kv_scale"].cpu().numpy().astype(np.float32)}
    return {"qa": host_bf16(lay["q"]), "kv": host_bf16(lay["kv"])}


class OraclePath:
    """The whole path for a list of query rows on the C++ oracle: indexer scores,
    streaming selection (flat, hierarchical or over entries), then the sparse
    attention of every layer. Page keys are pooled once, outside the timed
    part, as on the GPU."""

    def __init__(self, w, x, layers_host, fp8=False):
        import oracle as O
        self.O, self.w, self.x, self.layers, self.fp8 = O, w, x, layers_host, fp8
        self.kind = kind_of(w)
        if w.P and fp8:
            self.pk, self.ps = O.pool_pages_e4m3(x["k_idx_fp8"], x["k_scale"], x["seq_len"], w.P)
        elif w.P:
            self.pk = O.pool_pages(x["k_idx"], x["seq_len"], w.P)

    def run(self, rows):
        import numpy as np
        O, w, x = self.O, self.w, self.x
        budget = (w.k, w.sink, w.window)
        if self.fp8:
            q, k = x["q_idx_fp8"], x["k_idx_fp8"]
            kw = dict(fp8=True, q_scale=x["q_scale"], k_scale=x["k_scale"])
        else:
            q, k, kw = x["q_idx"], x["k_idx"], {}
        if self.kind == "compressed":
            idx, _ = O.index_compressed(q, x["w"], k, x["seq_len"], m=w.m, budget=w.k, sink=w.sink,
                                        window=w.window, **kw)
        elif w.P and self.fp8:
            idx, _ = O.index_hier_e4m3(q, x["q_scale"], x["w"], k, x["k_scale"], self.pk, self.ps, x["seq_len"], P=w.P,
                                       M=w.M, budget=w.k, sink=w.sink, window=w.window, rows=rows)
        elif w.P:
            idx, _ = O.index_hier(q, x["w"], k, self.pk, x["seq_len"], P=w.P, M=w.M, budget=w.k, sink=w.sink,
                                  window=w.window, rows=rows)
        else:
            sc = O.indexer_scores_rows(q, x["w"], k, x["seq_len"], rows, **kw)
            idx = np.full((w.B, w.T, w.k), -1, np.int32)
            for i, (b, t) in enumerate(rows):
                idx[b, t] = O.select_streaming_row(sc[i], int(x["seq_len"][b]) - w.T + t, *budget)
        for lay in self.layers:
            if "kv8" in lay:
                O.sparse_attention_e4m3_rows(lay["qa"], idx, rows, scale=w.scale, d_v=w.d_v, kv8=lay["kv8"],
                                             k_scale=lay["ks"])
            else:
                O.sparse_attention_rows(lay["qa"], idx, rows, scale=w.scale, d_v=w.d_v, kv=lay["kv"])

    def all_rows(self):
        return [(b, t) for b in range(self.w.B) for t in range(self.w.T)]


def time_oracle(op: OraclePath, rows, budget_s: float):
    """Repeat the rows until budget_s has passed (at least once): rows/s."""
    n, t0 = 0, time.perf_counter()
    while True:
        op.run(rows)
        n += len(rows)
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            return n / dt, n, dt


def cpu_baseline(op: OraclePath, budget_s: float = 12.0):
    import oracle as O
    w = op.w
    rows = op.all_rows()
    if op.kind == "prefill":                      # a stride of query rows (the full chunk is ~2e12 MACs)
        rows = [(0, t) for t in range(0, w.T, w.T // 32)]
    if op.kind == "compressed":
        rows = op.all_rows()
    O.set_threads(0)
    cores = O.threads()
    op.run(rows[:1])                               # warm the caches and pages
    v, n, dt = time_oracle(op, rows, budget_s)
    O.set_threads(1)
    try:
        v1, n1, dt1 = time_oracle(op, rows[:1] if op.kind != "compressed" else rows, min(budget_s / 2, 6.0))
    finally:
        O.set_threads(0)
    return {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} query rows ({len(rows)} per pass{', a stride of the chunk' if op.kind == 'prefill' else ''}"
                      f") through the whole path in {dt:.1f} s on {cores} threads",
            "one_thread": {"value": v1, "unit": UNIT, "sample": f"{n1} query rows in {dt1:.1f} s on 1 thread"}}


def run_reference(args, rank: int, world: int):
    """The C++ oracle as it stands on the host cores, same workload and metric."""
    if rank != 0:
        return 0
    if args.workload == "hier_sweep":
        print(json.dumps({"impl": "reference", "unavailable": "hier_sweep is a table of device timings (flat against "
                          "hierarchical indexing at four lengths); the oracle arm times single workloads, e.g. "
                          "--workload hier_decode_1m"}), flush=True)
        return 0
    import oracle as O
    from kv_indexing_b200 import inputs as I
    w = I.WORKLOADS[args.workload]
    x = host_inputs(w, args.seed, args.fp8)
    kv_w = I.entry_workload(w) if w.m else w
    layers = [I.make_attn_inputs(kv_w, args.seed, layer=li) for li in range(w.n_layers)]
    if not w.mla:   # our arm's cache has one row per token, V its first d_v columns: the same here
        for lay in layers:
            lay["kv"] = lay.pop("k")
            del lay["v"]
    if args.fp8_kv:   # the same per-token e4m3 quantisation the device path applies
        for lay in layers:
            lay["kv8"], lay["ks"] = I.quantize_e4m3_rows(I.bf16_bits_to_f32(lay.pop("kv")))
    op = OraclePath(w, x, layers, fp8=args.fp8)
    rows = op.all_rows()
    if op.kind == "prefill":
        rows = [(0, t) for t in range(0, w.T, w.T // 32)]
    O.set_threads(0)
    t0 = time.perf_counter()
    op.run(rows)
    per_pass = time.perf_counter() - t0
    # keep the whole --steps/--warmup run within a few minutes: each step runs
    # the batch, or a bounded sample of its rows when the batch is slower
    budget_step = 150.0 / max(1, args.steps + args.warmup)
    if per_pass > budget_step and len(rows) > 1:
        rows = rows[:max(1, int(len(rows) * budget_step / per_pass))]
    for _ in range(args.warmup):
        op.run(rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        op.run(rows)
    dt = time.perf_counter() - t0
    v = len(rows) * args.steps / dt
    sample = f"{len(rows)} of the {w.B * w.T} query rows per step, whole path, {O.threads()} threads"
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (the same seeded inputs as our arm's host generator)",
        "config": workload_config(w, parallelism="host threads", l2="n/a (host run)", fp8_indexer=bool(args.fp8),
                                  kv_cache="e4m3 (per-token fp32 scale)" if args.fp8_kv else "bf16"),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": O.threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------


def roofline(path, br, peaks, peak_src, fp8, torch, dev):
    w = path.w
    us = br[path.dominant]
    if path.kind == "prefill":
        achieved = path.roof_flops / (us * 1e-6) / 1e12
        peak, src = peaks["bf16_tflops"], peak_src + " bf16 burst (the indexer is timed in its own stage)"
        if fp8:
            fp8_peak = measure_fp8_peak(torch, dev)
            if fp8_peak:
                peak, src = fp8_peak, "e4m3 GEMM measured in this run (torch._scaled_mm 8192^3, best of 10)"
            else:
                peak, src = 2 * peaks["bf16_tflops"], peak_src + " bf16 burst x 2 (nominal e4m3 ratio)"
        traffic = kernel_traffic("indexer_" + w.name) if not fp8 else None
        return {"bound": "tensor", "kernel": path.roof_kernel, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "algorithmic_flops_per_launch": path.roof_flops,
                "launch_us": us, "peak_source": src}
    achieved = path.roof_bytes / (us * 1e-6) / 1e9
    traffic = None
    if path.kind == "flat" and not fp8:
        traffic = kernel_traffic("indexer_" + w.name)
    return {"bound": "hbm", "kernel": path.roof_kernel, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "algorithmic_bytes_per_launch": path.roof_bytes,
            "launch_us": us, "peak_source": peak_src + " HBM copy"}


def measure_fp8_peak(torch, dev):
    try:
        n = 8192
        a = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn).t()
        one = torch.tensor(1.0, device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        best = None
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(10):
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except Exception:
        return None


def step_bytes(path) -> float:
    w = path.w
    if path.kind == "prefill":
        return None
    if path.kind == "hier":
        ib = hier_index_bytes_per_query(w, path.fp8)
    elif path.kind == "group":
        return path.roof_bytes
    else:
        ib = indexer_bytes_per_query(w, path.fp8, w.L // w.m if w.m else w.L)
    return (ib + attention_bytes_per_query(w, path.kv8) + w.k * 4) * w.B * w.T


def run_workload(args, w, rank, world, dev, pg):
    import torch
    import torch.distributed as dist
    from kv_indexing_b200 import lsa as L

    seed = rank_seed(args.seed, rank)
    x = host_inputs(w, seed, args.fp8)
    path = Path(torch, L, w, x, dev, seed, args.fp8, kv8=args.fp8_kv)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.random_(0, 255)   # touch 256 MiB (> 126 MB L2)

    t = time_device(torch, path.stages, args.steps, args.warmup, flush, dev, pg, path.breakdown_stages)
    L.lsa_device_status()
    extra = dict(path.extra)
    if path.kind == "group":
        ti = time_device(torch, path.index_alone, max(10, args.steps // 4), 3, flush, dev, pg)
        extra["index_alone_us"] = ti["breakdown_us"]["index_alone"]
        extra["index_per_layer_amortised_us"] = ti["breakdown_us"]["index_alone"] / w.n_layers
    units = w.B * w.T * world
    value = units / (t["ms_per_step"] / 1000.0)
    peaks, peak_src = measured_peaks()
    roof = roofline(path, t["breakdown_us"], peaks, peak_src, args.fp8, torch, dev)
    sb = step_bytes(path)
    if sb:
        roof["step_frac_of_hbm_roofline"] = sb / (t["ms_per_step"] * 1e-3) / 1e9 / peaks["hbm_gbs"]
        roof["step_algorithmic_bytes"] = sb
    e2e = None if args.no_e2e else time_e2e(torch, path, max(20, min(args.steps, 100)), flush, dev, pg)
    L.lsa_device_status()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        layers_host = [host_layer(l) for l in path.layers]
        del flush_buf
        torch.cuda.empty_cache()
        cpu = cpu_baseline(OraclePath(w, x, layers_host, fp8=args.fp8))
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if args.fp8 else "bf16",
            "data": "synthetic (seeded N(0,1) bf16 indexer inputs, U(0,1) head weights and 1% planted needles from "
                    "the host generator; latent KV and attention queries drawn on the device with a seeded "
                    "generator)",
            "config": workload_config(w, parallelism=f"replicas x{world} (independent batches)",
                                      fp8_indexer=bool(args.fp8),
                                      kv_cache="e4m3 (per-token fp32 scale)" if args.fp8_kv else "bf16"),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": (t["launches_per_step"] or 0) * args.steps,
            "launches_per_step": t["launches_per_step"],
            "breakdown_us": t["breakdown_us"],
            "plain_launches": {"ms_per_step": t["plain_ms_per_step"],
                               "value": units / (t["plain_ms_per_step"] / 1000.0)},
            "graph_note": "value: one CUDA graph per step with events only around it (consecutive kernels overlap "
                          "their launch); breakdown_us: a second graph with events between the stages (the "
                          "indexing call split into scores alone and the selection)",
            "tokens_scanned_per_s": value * w.L, "clocks": t["clocks"], **extra,
        }
        print(json.dumps(line), flush=True)
    return 0


def run_sweep(args, rank, world, dev, pg):
    """Flat against hierarchical indexing on identical inputs (B=2, P=64, M=256,
    k=2048), L = 64K .. 1M: the indexing call alone and the whole step."""
    import torch
    from kv_indexing_b200 import inputs as I
    from kv_indexing_b200 import lsa as L

    seed = rank_seed(args.seed, rank)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.random_(0, 255)

    peaks, peak_src = measured_peaks()
    table = []
    K = max(10, min(args.steps, 50))
    for Lc in SWEEP_L:
        wh = I.scaled(I.WORKLOADS["hier_decode_1m"], L=Lc, name=f"hier_decode_{Lc // 1024}k")
        wf = I.scaled(I.WORKLOADS["flat_decode_1m"], L=Lc, name=f"flat_decode_{Lc // 1024}k")
        x = host_inputs(wh, seed)                 # identical for both (same seed and shapes)
        ph = Path(torch, L, wh, x, dev, seed, False)
        pf = Path(torch, L, wf, x, dev, seed, False, layers=ph.layers)   # the same latent KV and queries
        th = time_device(torch, ph.stages, K, 3, flush, dev, pg)
        tf = time_device(torch, pf.stages, K, 3, flush, dev, pg)
        flat_index = tf["breakdown_us"]["index"]
        hier_index = th["breakdown_us"]["hier_index"]
        table.append({
            "L": Lc, "flat_index_us": flat_index, "hier_index_us": hier_index,
            "index_speedup_hier_over_flat": flat_index / hier_index,
            "flat_step_us": 1000 * tf["ms_per_step"], "hier_step_us": 1000 * th["ms_per_step"],
            "step_speedup_hier_over_flat": tf["ms_per_step"] / th["ms_per_step"],
            "flat_index_frac_of_hbm": indexer_bytes_per_query(wf) * wf.B / (flat_index * 1e-6) / 1e9
            / peaks["hbm_gbs"],
            "hier_index_frac_of_hbm": hier_index_bytes_per_query(wh) * wh.B / (hier_index * 1e-6) / 1e9
            / peaks["hbm_gbs"],
            "clocks_sm_mhz": th["clocks"]["sm_mhz"], "clock_reasons": sorted(set(th["clocks"]["reasons"]) |
                                                                             set(tf["clocks"]["reasons"])),
        })
        del ph, pf
        torch.cuda.empty_cache()
    last = table[-1]
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": 2 * world / (last["hier_step_us"] * 1e-6), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": 3, "ms_per_step": last["hier_step_us"] / 1000, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "hier_sweep", "B": 2, "P": 64, "M": 256, "k": 2048, "L": list(SWEEP_L),
                       "l2": "flushed between timed steps"},
            "sweep": table, "peak_source": peak_src,
            "note": "index = the indexing call(s) only (flat: scores + top-k; hierarchical: page scores, recall, "
                    "fine scores, top-k; page pooling is once per filled page, outside); step = index + attention",
        }), flush=True)
    return 0


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist

    from kv_indexing_b200 import inputs as I
    from kv_indexing_b200 import lsa as L

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
        pg = True
    L.load()
    try:
        if args.workload == "hier_sweep":
            return run_sweep(args, rank, world, dev, pg)
        return run_workload(args, I.WORKLOADS[args.workload], rank, world, dev, pg)
    finally:
        if pg:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
