#!/usr/bin/env python
"""Benchmark of the LSA decode hot path on B200.

One step = one pass of the whole path over one batch: lightning-indexer scores
(tcgen05) -> streaming top-k -> sparse MLA attention (+ split combine), on the
flat-decode workload (8 sequences x 131072 cached tokens, one query each, top-k
2048 = sink 64 + window 960 + 1024 dynamic; 128 query heads, d_qk 576 / d_v 512)
unless --workload says otherwise. Inputs are seeded synthetic data resident in
HBM; L2 is flushed (256 MiB write) between timed steps, outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--fp8]

Workloads (kv_indexing_b200.inputs.WORKLOADS): flat_decode_128k (default, the
headline), hier_decode_1m (hierarchical indexing at 1M tokens; page pooling
timed once, outside the step), cli_group_256k / cli_group_256k_flat (one
indexing pass feeding two layers), prefill_64k (4096 causal queries; --fp8 for
e4m3 indexer inputs), compressed_decode_1m (indexing over 262144 entries of 4
tokens each, then attention over the 2048 chosen compressed latent entries;
--fp8 for e4m3 entry keys). Long KV caches for timing are drawn on the device with
torch's seeded generator; the indexer inputs come from the seeded host
generator (needles included).

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


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="flat_decode_128k")
    p.add_argument("--seed", type=int, default=1)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--fp8", action="store_true", help="prefill: e4m3 indexer keys and queries")
    return p.parse_args()


# ---------------------------------------------------------------------------
# algorithmic work per query (what the method must move), used for the roofline
# ---------------------------------------------------------------------------


def indexer_bytes_per_query(w) -> int:
    """Keys streamed once + the query's indexer vectors and head weights."""
    return w.L * w.d * 2 + w.H * w.d * 2 + w.H * 4


def attention_bytes_per_query(w) -> int:
    """Gathered latent KV rows + q + o."""
    return w.k * w.d_qk * 2 + w.Hq * w.d_qk * 2 + w.Hq * w.d_v * 2


def step_bytes_per_query(w) -> int:
    return indexer_bytes_per_query(w) + attention_bytes_per_query(w) + w.k * 4


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


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
    src = os.path.join(ROOT, ent["source_file"])
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
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


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_query(O, w, x, a, b):
    """The whole path for query (b, 0) on the CPU oracle."""
    rows = [(b, 0)]
    sc = O.indexer_scores(x["q_idx"], x["w"], x["k_idx"], x["seq_len"], rows=rows)
    pos = int(x["seq_len"][b]) - 1
    idx = O.select_streaming_row(sc[b, 0], pos, w.k, w.sink, w.window)
    ii = idx[None, None, :]
    qa = a["qa"][b:b + 1]
    kv = a["kv"][b:b + 1]
    O.sparse_attention(qa, ii, x["seq_len"][b:b + 1], scale=w.scale, d_v=w.d_v, kv=kv)


def time_oracle(w, x, a, budget_s: float = 12.0, max_queries=None):
    import oracle as O
    n, t0 = 0, time.perf_counter()
    total = w.B * w.T if max_queries is None else max_queries
    while n < total:
        oracle_query(O, w, x, a, n % w.B)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return n / dt, n, dt


def run_reference(args, rank: int, world: int):
    """The oracle as it stands on the host cores: one query per step."""
    if rank != 0:
        return 0
    from kv_indexing_b200 import inputs as I
    import oracle as O
    w = I.WORKLOADS[args.workload]
    x = I.make_indexer_inputs(w, args.seed)
    a = I.make_attn_inputs(w, args.seed)
    for i in range(args.warmup):
        oracle_query(O, w, x, a, i % w.B)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_query(O, w, x, a, i % w.B)
    dt = time.perf_counter() - t0
    v = args.steps / dt
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, sampled="one query of the batch per step"),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} single-query steps of the {w.B}-query batch"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, **extra):
    c = {"workload": w.name, "B": w.B, "L": w.L, "T": w.T, "H_I": w.H, "d_I": w.d, "k": w.k, "sink": w.sink,
         "window": w.window, "Hq": w.Hq, "d_qk": w.d_qk, "d_v": w.d_v, "P": w.P, "M": w.M,
         "n_layers": w.n_layers, "entry_tokens_m": w.m,
         "l2": "flushed between timed steps (256 MiB write, outside the timed events)"}
    c.update(extra)
    return c


# ---------------------------------------------------------------------------
# other workloads: a generic stage timer over one CUDA graph per step
# ---------------------------------------------------------------------------


def time_stages(torch, stages, K, warmup, flush, dev, pg):
    """stages: [(name, fn(stream))]. One graph per step with external events
    between the stages; L2 flushed between steps, outside the events."""
    import torch.distributed as dist
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, warmup)):
        flush()
        for _, fn in stages:
            fn(stream)
    torch.cuda.synchronize()
    n = len(stages)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n + 1)]
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
        s = torch.cuda.current_stream(dev)
        ev[0].record(s)
        for i, (_, fn) in enumerate(stages):
            fn(s)
            ev[i + 1].record(s)
    torch.cuda.synchronize()
    for _ in range(3):
        flush()
        g.replay()
    torch.cuda.synchronize()
    per = [[] for _ in range(n)]
    tot = []
    if pg:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        for _ in range(K):
            flush()
            g.replay()
            torch.cuda.synchronize()
            for i in range(n):
                per[i].append(ev[i].elapsed_time(ev[i + 1]))
            tot.append(ev[0].elapsed_time(ev[n]))
    torch.cuda.synchronize()
    if pg:
        dist.barrier()
    total_ms = max_over_ranks(float(sum(tot)), dev, pg)
    del g
    return {name: 1000 * sum(per[i]) / K for i, (name, _) in enumerate(stages)}, total_ms / K, clk.summary()


def device_bf16_normal(torch, shape, seed, dev):
    """Seeded N(0,1) bf16 drawn on the device (timing inputs for long KV caches)."""
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)


def run_workload(args, w, rank, world, dev, pg):
    import numpy as np
    import torch
    import torch.distributed as dist

    from kv_indexing_b200 import inputs as I
    from kv_indexing_b200 import lsa as L

    seed = rank_seed(args.seed, rank)
    if w.m:
        # compressed entries: the indexer's keys are the entry keys [B, L/m, d]
        x = I.make_compressed_inputs(w, seed)
        x["k_idx"] = x.pop("entry_keys")
        if "entry_keys_fp8" in x:
            x["k_idx_fp8"] = x.pop("entry_keys_fp8")
    else:
        x = I.make_indexer_inputs(w, seed)
    kv_rows = w.L // w.m if w.m else w.L

    def up(arr, kind):
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16) if kind == "bf16" else arr)
        t = t.view(torch.bfloat16) if kind == "bf16" else t
        return t.to(dev)

    q, k, wt, sl = up(x["q_idx"], "bf16"), up(x["k_idx"], "bf16"), up(x["w"], "f32"), up(x["seq_len"], "i32")
    B, T = w.B, w.T
    budget = (w.k, w.sink, w.window)
    layers = []
    for li in range(w.n_layers):
        qa = device_bf16_normal(torch, (B, T, w.Hq, w.d_qk), 7919 * seed + 2 * li, dev)
        kv = device_bf16_normal(torch, (B, kv_rows, w.d_qk), 7919 * seed + 2 * li + 1, dev)
        layers.append({"q": qa, "kv": kv, "scale": w.scale, "d_v": w.d_v})
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.random_(0, 255)

    peaks, peak_src = measured_peaks()
    idx = torch.empty((B, T, w.k), dtype=torch.int32, device=dev)
    outs = [torch.empty((B, T, w.Hq, w.d_v), dtype=torch.bfloat16, device=dev) for _ in range(w.n_layers)]
    extra = {}
    ai = L.attn_in(layers[0]["q"], sl, w.scale, kv=layers[0]["kv"], d_v=w.d_v)
    attn_ws = torch.empty(max(256, L.workspace_size(L.LSA_OP_SPARSE_ATTN, attn=ai, budget=(w.k, 0, 0))),
                          dtype=torch.uint8, device=dev)

    def attn_stage(li):
        lay = layers[li]
        return lambda s: L.lsa_sparse_attn(lay["q"], idx, sl, w.scale, kv=lay["kv"], d_v=w.d_v, out=outs[li],
                                           workspace=attn_ws, stream=s)

    if w.m:
        kind = "compressed"
        qk = dict(q=q, k=k)
        if args.fp8:
            qk = dict(q=up(x["q_idx_fp8"], "u8").view(torch.float8_e4m3fn),
                      k=up(x["k_idx_fp8"], "u8").view(torch.float8_e4m3fn),
                      q_scale=up(x["q_scale"], "f32"), k_scale=up(x["k_scale"], "f32"))
        ii = L.indexer_in(qk["q"], wt, qk["k"], sl, qk.get("q_scale"), qk.get("k_scale"), m=w.m)
        cws = torch.empty(max(256, L.workspace_size(L.LSA_OP_INDEX_COMPRESSED, indexer=ii, budget=budget, m=w.m)),
                          dtype=torch.uint8, device=dev)
        # one query per sequence (decode): its entry position is seq_len // m - 1
        sl_e = torch.div(sl, w.m, rounding_mode="floor").to(torch.int32)
        lay = layers[0]
        ai_c = L.attn_in(lay["q"], sl_e, w.scale, kv=lay["kv"], d_v=w.d_v, stream_budget=budget)
        cattn_ws = torch.empty(max(256, L.workspace_size(L.LSA_OP_SPARSE_ATTN, attn=ai_c, budget=(w.k, 0, 0))),
                               dtype=torch.uint8, device=dev)
        stages = [("index_compressed", lambda s: L.lsa_index_compressed(
                      qk["q"], wt, qk["k"], sl, w.m, budget, q_scale=qk.get("q_scale"), k_scale=qk.get("k_scale"),
                      idx=idx, workspace=cws, stream=s)),
                  ("attention", lambda s: L.lsa_sparse_attn(lay["q"], idx, sl_e, w.scale, kv=lay["kv"], d_v=w.d_v,
                                                            out=outs[0], workspace=cattn_ws, stream_budget=budget,
                                                            stream=s))]
    elif w.T > 1:
        kind = "prefill"
        qk = dict(q=q, k=k)
        if args.fp8:
            if "k_idx_fp8" not in x:
                raise SystemExit(f"workload {w.name} has no e4m3 indexer inputs")
            qk = dict(q=up(x["q_idx_fp8"], "u8").view(torch.float8_e4m3fn),
                      k=up(x["k_idx_fp8"], "u8").view(torch.float8_e4m3fn),
                      q_scale=up(x["q_scale"], "f32"), k_scale=up(x["k_scale"], "f32"))
        ii = L.indexer_in(qk["q"], wt, qk["k"], sl, qk.get("q_scale"), qk.get("k_scale"))
        scores = torch.empty((B, T, w.L), dtype=torch.float32, device=dev)
        sel_ws = torch.empty(max(256, L.workspace_size(L.LSA_OP_SELECT, budget=budget, B=B, T=T, L_max=w.L)),
                             dtype=torch.uint8, device=dev)
        stages = [("indexer", lambda s: L.lsa_index_flat(qk["q"], wt, qk["k"], sl, budget,
                                                         q_scale=qk.get("q_scale"), k_scale=qk.get("k_scale"),
                                                         scores_out=scores, with_idx=False, stream=s)),
                  ("select", lambda s: L.lsa_select_streaming(scores, sl, budget, idx=idx, workspace=sel_ws,
                                                              stream=s)),
                  ("attention", attn_stage(0))]
    elif w.n_layers > 1:
        kind = "group"
        page_keys = L.lsa_pool_pages(k, sl, w.P) if w.P else None
        ii = L.indexer_in(q, wt, k, sl)
        ais = [L.attn_in(l["q"], sl, w.scale, kv=l["kv"], d_v=w.d_v) for l in layers]
        ws = torch.empty(max(256, L.workspace_size(L.LSA_OP_LAYER_GROUP, indexer=ii, attn=ais, budget=budget,
                                                   P=w.P, M=w.M, n_layers=w.n_layers)), dtype=torch.uint8, device=dev)
        stages = [("group", lambda s: L.lsa_layer_group(q, wt, k, sl, budget, layers, P=w.P, M=w.M,
                                                        page_keys=page_keys, outs=outs, idx=idx, workspace=ws,
                                                        stream=s))]
    else:
        kind = "hier"
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        page_keys = torch.zeros((B, w.L // w.P, w.d), dtype=torch.bfloat16, device=dev)
        e0.record()
        L.lsa_pool_pages(k, sl, w.P, page_keys=page_keys)
        e1.record()
        torch.cuda.synchronize()
        extra["page_pooling_once_us"] = 1000 * e0.elapsed_time(e1)
        ii = L.indexer_in(q, wt, k, sl)
        ws = torch.empty(max(256, L.workspace_size(L.LSA_OP_INDEX_HIER, indexer=ii, budget=budget, P=w.P, M=w.M)),
                         dtype=torch.uint8, device=dev)
        stages = [("hier_index", lambda s: L.lsa_index_hier(q, wt, k, sl, page_keys, w.P, w.M, budget, idx=idx,
                                                            workspace=ws, stream=s)),
                  ("attention", attn_stage(0))]

    br, ms_per_step, clocks = time_stages(torch, stages, args.steps, args.warmup, flush, dev, pg)
    L.lsa_device_status()
    units = B * T * world
    value = units / (ms_per_step / 1000.0)

    # roofline of the dominant stage
    if kind == "prefill":
        pos = np.arange(w.L - w.T, w.L, dtype=np.float64)
        flops = 2.0 * w.H * w.d * float(np.sum(pos + 1)) * B
        us = br["indexer"]
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * (2.0 if args.fp8 else 1.0)
        roof = {"bound": "tensor", "kernel": "indexer (tcgen05 score GEMM over causal tiles, fused epilogue)",
                "achieved": flops / (us * 1e-6) / 1e12, "peak": peak, "unit": "TFLOP/s",
                "frac": flops / (us * 1e-6) / 1e12 / peak, "traffic": None, "algorithmic_flops_per_launch": flops,
                "launch_us": us, "peak_source": peak_src + (" bf16 sustained x 2 (e4m3 nominal ratio)" if args.fp8
                                                             else " bf16 sustained")}
    elif kind == "compressed":
        n_e = w.L // w.m
        byts = (n_e * w.d * (1 if args.fp8 else 2) + (n_e * 4 if args.fp8 else 0) + w.H * w.d * 2 + w.H * 4) * B * T
        us = br["index_compressed"]
        roof = {"bound": "hbm", "kernel": "compressed-entry indexing call (entry scores, streaming top-k)",
                "achieved": byts / (us * 1e-6) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": byts / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], "traffic": None,
                "algorithmic_bytes_per_launch": byts, "launch_us": us, "peak_source": peak_src}
    elif kind == "group":
        if w.P:
            ib = (w.L // w.P) * w.d * 2 + w.M * w.P * w.d * 2
        else:
            ib = indexer_bytes_per_query(w)
        byts = (ib + w.n_layers * attention_bytes_per_query(w)) * B * T
        us = br["group"]
        roof = {"bound": "hbm", "kernel": "layer-group call (one indexing pass + %d attention layers)" % w.n_layers,
                "achieved": byts / (us * 1e-6) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": byts / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], "traffic": None,
                "algorithmic_bytes_per_launch": byts, "launch_us": us, "peak_source": peak_src}
    else:
        byts = ((w.L // w.P) * w.d * 2 + w.M * w.P * w.d * 2) * B * T
        us = br["hier_index"]
        roof = {"bound": "hbm", "kernel": "hierarchical indexing call (page scores, recall, fine scores, top-k)",
                "achieved": byts / (us * 1e-6) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": byts / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], "traffic": None,
                "algorithmic_bytes_per_launch": byts, "launch_us": us, "peak_source": peak_src}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if args.fp8 else "bf16",
            "data": "synthetic (seeded N(0,1) bf16 indexer inputs with 1% needles from the host generator; "
                    "latent KV and attention queries drawn on the device with a seeded generator)",
            "config": workload_config(w, parallelism=f"replicas x{world} (independent batches)",
                                      fp8_indexer=bool(args.fp8)),
            "roofline": roof, "cpu_baseline": None, "e2e": None, "breakdown_us": br, **extra,
            "tokens_scanned_per_s": value * w.L, "clocks": clocks,
            "note": "extra workload line; the headline, e2e and CPU baseline are on flat_decode_128k",
        }
        print(json.dumps(line), flush=True)
    if pg:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import numpy as np
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
    w = I.WORKLOADS[args.workload]
    if w.P or w.m or w.n_layers > 1 or w.T > 1 or args.fp8:
        return run_workload(args, w, rank, world, dev, pg)
    seed = rank_seed(args.seed, rank)                   # each rank its own batch
    x = I.make_indexer_inputs(w, seed)
    a = I.make_attn_inputs(w, seed)

    def up(arr, kind):
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16) if kind == "bf16" else arr)
        t = t.view(torch.bfloat16) if kind == "bf16" else t
        return t.to(dev)

    q, k, wt = up(x["q_idx"], "bf16"), up(x["k_idx"], "bf16"), up(x["w"], "f32")
    sl = up(x["seq_len"], "i32")
    qa, kv = up(a["qa"], "bf16"), up(a["kv"], "bf16")
    B, T = w.B, w.T
    budget = (w.k, w.sink, w.window)
    scores = torch.empty((B, T, w.L), dtype=torch.float32, device=dev)
    idx = torch.empty((B, T, w.k), dtype=torch.int32, device=dev)
    out = torch.empty((B, T, w.Hq, w.d_v), dtype=torch.bfloat16, device=dev)
    ai = L.attn_in(qa, sl, w.scale, kv=kv, d_v=w.d_v, stream_budget=budget)
    attn_ws_n = L.workspace_size(L.LSA_OP_SPARSE_ATTN, attn=ai, budget=(w.k, 0, 0))
    attn_ws = torch.empty(max(attn_ws_n, 256), dtype=torch.uint8, device=dev)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flat_ws = torch.empty(L.workspace_size(L.LSA_OP_INDEX_FLAT, indexer=L.indexer_in(q, wt, k, sl), budget=budget),
                          dtype=torch.uint8, device=dev)
    sel_ws = torch.empty(max(256, L.workspace_size(L.LSA_OP_SELECT, budget=budget, B=B, T=T, L_max=w.L)),
                         dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def k_index():
        L.lsa_index_flat(q, wt, k, sl, budget, scores_out=scores, with_idx=False, stream=stream)

    def k_select():
        L.lsa_select_streaming(scores, sl, budget, idx=idx, workspace=sel_ws, stream=stream)

    def k_attn():
        L.lsa_sparse_attn(qa, idx, sl, w.scale, kv=kv, d_v=w.d_v, out=out, workspace=attn_ws, stream=stream,
                          stream_budget=budget)

    def flush():
        flush_buf.random_(0, 255)   # touch 256 MiB (> 126 MB L2)

    for _ in range(max(3, args.warmup)):
        flush()
        k_index(); k_select(); k_attn()
    torch.cuda.synchronize()
    L.lsa_device_status()

    # One CUDA graph per step. The timed graph has events only around the whole
    # step, so consecutive kernels may overlap their launch (programmatic
    # dependent launch); a second graph with events between the stages gives
    # the per-stage breakdown (stages then run back to back).
    def capture(stage_events):
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
            s = torch.cuda.current_stream(dev)
            ev[0].record(s)
            L.lsa_index_flat(q, wt, k, sl, budget, scores_out=scores, with_idx=False, stream=s)
            if stage_events:
                ev[1].record(s)
            L.lsa_select_streaming(scores, sl, budget, idx=idx, workspace=sel_ws, stream=s)
            if stage_events:
                ev[2].record(s)
            L.lsa_sparse_attn(qa, idx, sl, w.scale, kv=kv, d_v=w.d_v, out=out, workspace=attn_ws, stream=s,
                              stream_budget=budget)
            ev[3].record(s)
        torch.cuda.synchronize()
        for _ in range(3):
            flush()
            g.replay()
        torch.cuda.synchronize()
        return g, ev

    g, ev = capture(False)
    gb, evb = capture(True)

    K = args.steps
    t_step, t_idx, t_sel, t_att = [], [], [], []
    if pg:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        for _ in range(K):
            flush()
            g.replay()
            torch.cuda.synchronize()
            t_step.append(ev[0].elapsed_time(ev[3]))
    torch.cuda.synchronize()
    if pg:
        dist.barrier()
    for _ in range(K):
        flush()
        gb.replay()
        torch.cuda.synchronize()
        t_idx.append(evb[0].elapsed_time(evb[1]))
        t_sel.append(evb[1].elapsed_time(evb[2]))
        t_att.append(evb[2].elapsed_time(evb[3]))
    torch.cuda.synchronize()
    L.lsa_device_status()
    total_ms = max_over_ranks(float(sum(t_step)), dev, pg)
    ms_per_step = total_ms / K
    units = B * T * world
    value = units / (ms_per_step / 1000.0)

    # end to end through the public API with host buffers: per step copy the
    # step's queries in (indexer q and w, attention q), read o and idx back
    e2e = None
    if not args.no_e2e:
        hq = torch.from_numpy(x["q_idx"].view(np.int16)).view(torch.bfloat16).pin_memory()
        hw = torch.from_numpy(x["w"]).pin_memory()
        hqa = torch.from_numpy(a["qa"].view(np.int16)).view(torch.bfloat16).pin_memory()
        ho = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
        hi = torch.empty(idx.shape, dtype=torch.int32).pin_memory()
        dq, dw, dqa = torch.empty_like(q), torch.empty_like(wt), torch.empty_like(qa)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hw, hqa))
        d2h = ho.numel() * ho.element_size() + hi.numel() * hi.element_size()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_ms = []
        for i in range(3 + K):
            flush()
            e0.record(stream)
            dq.copy_(hq, non_blocking=True); dw.copy_(hw, non_blocking=True); dqa.copy_(hqa, non_blocking=True)
            ix = L.lsa_index_flat(dq, dw, k, sl, budget, idx=idx, workspace=flat_ws, stream=stream)
            L.lsa_sparse_attn(dqa, ix, sl, w.scale, kv=kv, d_v=w.d_v, out=out, workspace=attn_ws, stream=stream,
                              stream_budget=budget)
            ho.copy_(out, non_blocking=True); hi.copy_(idx, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= 3:
                e2e_ms.append(e0.elapsed_time(e1))
        em = max_over_ranks(sum(e2e_ms) / len(e2e_ms), dev, pg)
        e2e = {"value": units / (em / 1000.0), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": em,
               "note": "KV and indexer-key caches resident; per step the new queries go in and o, idx come out"}

    peaks, peak_src = measured_peaks()
    idx_us = 1000 * sum(t_idx) / K
    idx_bytes = indexer_bytes_per_query(w) * B * T
    achieved = idx_bytes / (idx_us * 1e-6) / 1e9
    roof = {"bound": "hbm", "kernel": "indexer (tcgen05 score GEMM + fused epilogue)", "achieved": achieved,
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
            "traffic": kernel_traffic("indexer_flat_decode_128k"),
            "algorithmic_bytes_per_launch": idx_bytes, "launch_us": idx_us, "peak_source": peak_src,
            "step_frac_of_hbm_roofline": (step_bytes_per_query(w) * B * T / (ms_per_step * 1e-3) / 1e9)
            / peaks["hbm_gbs"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, dt = time_oracle(w, x, a)
        cpu = {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n} of {B * T} queries of the batch, whole path, {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16, U(0,1) head weights, 1% planted needles)",
            "config": workload_config(w, parallelism=f"replicas x{world} (independent batches)"),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": 4 * K,
            "breakdown_us": {"indexer": idx_us, "select": 1000 * sum(t_sel) / K, "attention": 1000 * sum(t_att) / K,
                             "note": "stages timed back to back (events between them); the value's step lets "
                                     "consecutive kernels overlap their launch"},
            "tokens_scanned_per_s": value * w.L,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    del g, gb
    if pg:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
