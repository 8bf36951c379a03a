"""Host logic of the multi-GPU bench path on CPU: two gloo ranks.

Each rank decodes its own independent sequence (weak scaling, no data-path
collective); the only collective is the max-over-ranks reduction of the
timings, which every rank calls in the same order.
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


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # every rank makes the same reductions in the same order
        t = bench.max_over_ranks(10.0 + rank, world, device="cpu")
        u = bench.max_over_ranks(5.0 - rank, world, device="cpu")
        wl = bench.make_workload(4096, rank, device="cpu")
        q.put((rank, t, u, float(wl.q.sum())))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_max_timing_and_independent_sequences():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]          # slowest rank's time everywhere
    assert [r[2] for r in res] == [5.0, 5.0]
    assert res[0][3] != res[1][3]                        # each rank its own sequence
