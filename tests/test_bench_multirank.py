"""Multi-rank host logic of bench.py on CPU: two gloo ranks (one process per
rank, as torchrun launches them). The timed value is the slowest rank's time,
every rank draws its own batch, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(1.5 + rank, torch.device("cpu"), True)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(1, rank))
        class A:
            impl, workload, seed, steps, warmup, gpus = "reference", "tiny_l2k", 1, 1, 0, world
        ref_rc = bench.run_reference(A, rank, world) if rank != 0 else None
        q.put((rank, t, seeds, ref_rc))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_distinct_batches_reference_on_rank0_only():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, s0, _), (r1, t1, s1, rc1) = res
    assert t0 == t1 == 2.5                       # both ranks report the slower rank's time
    assert len(set(s0)) == 2 and s0 == s1        # each rank its own seeded batch
    assert rc1 == 0                              # non-zero ranks leave the reference arm at once
