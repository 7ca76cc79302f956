"""Replica aggregation of bench.py over several processes (CPU, gloo, world 2).

The path has no exchange step, so multi-GPU runs are independent replicas; the
only cross-rank logic is the timing barrier and the max-time / summed-work
reduction, tested here on CPU with the gloo backend.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.0, 5.0][rank]
        byts = [100.0, 250.0][rank]
        toks = [7.0, 11.0][rank]
        dist.barrier()
        res = bench.reduce_over_ranks(ms, byts, toks, torch.device("cpu"))
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_two_processes():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        assert out[r] == (5.0, 350.0, 18.0)


def test_single_process_is_identity():
    import bench
    assert bench.reduce_over_ranks(2.5, 10.0, 3.0, torch.device("cpu")) == (2.5, 10.0, 3.0)


def test_replica_plan_exceeds_four_l2():
    import bench
    from turboquant_kv_cache_rht_b200 import workloads as wl
    l2 = 126 << 20
    for name in ("gqa", "qjl", "long", "serving", "tiny"):
        w = wl.WORKLOADS[name]
        p = bench.replica_plan(w, bench.default_steps_total(), l2)
        per = sum(p["lengths"]) * w.kv_heads * bench.token_bytes(w)
        assert p["replicas"] * per > 4 * l2 or p["replicas"] == 64
        assert p["capacity"] % 16 == 0 and p["capacity"] >= p["max_ctx"] >= max(p["lengths"])
