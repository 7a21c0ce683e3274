#!/usr/bin/env python
"""Benchmark of the LSA decode hot path on B200.

One step = one pass of the whole path over one batch: lightning-indexer scores
(tcgen05) -> streaming top-k -> sparse MLA attention (+ split combine), on the
flat-decode workload (8 sequences x 131072 cached tokens, one query each, top-k
2048 = sink 64 + window 960 + 1024 dynamic; 128 query heads, d_qk 576 / d_v 512)
unless --workload says otherwise. Inputs are seeded synthetic data resident in
HBM; L2 is flushed (256 MiB write) between timed steps, outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

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
         "n_layers": w.n_layers, "l2": "flushed between timed steps (256 MiB write, outside the timed events)"}
    c.update(extra)
    return c


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
    if w.P or w.n_layers > 1 or w.T > 1:
        raise SystemExit(f"bench.py times the flat decode step; workload {w.name} is covered by the tests")
    seed = args.seed + 1000 * rank                       # each rank its own batch
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
    ai = L.attn_in(qa, sl, w.scale, kv=kv, d_v=w.d_v)
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
        L.lsa_sparse_attn(qa, idx, sl, w.scale, kv=kv, d_v=w.d_v, out=out, workspace=attn_ws, stream=stream)

    def flush():
        flush_buf.random_(0, 255)   # touch 256 MiB (> 126 MB L2)

    for _ in range(max(3, args.warmup)):
        flush()
        k_index(); k_select(); k_attn()
    torch.cuda.synchronize()
    L.lsa_device_status()

    # one CUDA graph per step, with timing events between the kernels
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
        s = torch.cuda.current_stream(dev)
        ev[0].record(s)
        L.lsa_index_flat(q, wt, k, sl, budget, scores_out=scores, with_idx=False, stream=s)
        ev[1].record(s)
        L.lsa_select_streaming(scores, sl, budget, idx=idx, workspace=sel_ws, stream=s)
        ev[2].record(s)
        L.lsa_sparse_attn(qa, idx, sl, w.scale, kv=kv, d_v=w.d_v, out=out, workspace=attn_ws, stream=s)
        ev[3].record(s)
    torch.cuda.synchronize()
    for _ in range(3):
        flush()
        g.replay()
    torch.cuda.synchronize()

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
            t_idx.append(ev[0].elapsed_time(ev[1]))
            t_sel.append(ev[1].elapsed_time(ev[2]))
            t_att.append(ev[2].elapsed_time(ev[3]))
            t_step.append(ev[0].elapsed_time(ev[3]))
    torch.cuda.synchronize()
    if pg:
        dist.barrier()
    L.lsa_device_status()
    total_ms = float(sum(t_step))
    if pg:
        tt = torch.tensor([total_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        total_ms = float(tt.item())
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
            L.lsa_sparse_attn(dqa, ix, sl, w.scale, kv=kv, d_v=w.d_v, out=out, workspace=attn_ws, stream=stream)
            ho.copy_(out, non_blocking=True); hi.copy_(idx, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= 3:
                e2e_ms.append(e0.elapsed_time(e1))
        em = sum(e2e_ms) / len(e2e_ms)
        if pg:
            tt = torch.tensor([em], device=dev, dtype=torch.float64)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            em = float(tt.item())
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
            "breakdown_us": {"indexer": idx_us, "select": 1000 * sum(t_sel) / K, "attention": 1000 * sum(t_att) / K},
            "tokens_scanned_per_s": value * w.L,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    del g
    if pg:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
