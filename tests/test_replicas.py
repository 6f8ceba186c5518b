"""Multi-process plumbing of bench.py's replica mode on CPU (gloo,
world size 2): every rank reports the slowest rank's time, and replicas draw
different inputs.  The decode path itself has no collective."""
import datetime
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


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from sparse_decode_attention_saga_b200.workload import CONFIGS, make_queries
        slowest = bench.max_over_ranks(1.5 + rank, world, device="cpu")
        bench.barrier(world)
        q = make_queries(CONFIGS["tiny"].scaled(steps=1), seed=0 + rank)
        digest = float(q.float().sum())
        results.put((rank, slowest, digest))
    finally:
        dist.destroy_process_group()


def test_replicas_report_slowest_rank_and_draw_distinct_inputs():
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(results.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [2.5, 2.5]
    assert got[0][2] != got[1][2]
