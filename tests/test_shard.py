"""Kv-head sharding of one decode step over ranks (host logic, gloo on the CPU).

The step shards by kv head with no exchange inside it; the output rows of every
rank are gathered at the end.  Each rank here runs a stand-in step over its own
kv heads -- the oracle's pipeline (replica bounds, top-k, float64 entmax
attention) on the rank's slice of the query -- so the gathered output must equal,
bit for bit, the same pipeline run by one rank over every kv head.
"""
import math
import os
import socket
from dataclasses import replace

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import attend, replica, select
from sparse_long_context_min_b200 import workloads
from sparse_long_context_min_b200.shard import HeadShardedStep, kv_head_range, shard


def test_kv_head_ranges_partition_the_heads():
    for H in (1, 2, 5, 8, 32):
        for world in range(1, H + 1):
            ranges = [kv_head_range(H, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))       # contiguous, no overlap
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        kv_head_range(4, 8, 0)                 # more ranks than kv heads
    q = torch.arange(2 * 32 * 3).reshape(2, 32, 3)
    assert torch.equal(shard(q, 1, 2, 4, per_head=4), q[:, 8:16])


def _workload():
    cfg = replace(workloads.config(2), B=2, lengths=[2048 + 17, 1500])
    return workloads.Workload(cfg, device="cpu")


class OracleStep:
    """Stand-in for a rank's DecodeStep: the oracle pipeline over kv heads [g0, g1)."""

    def __init__(self, wl, g0, g1):
        self.wl, self.g0, self.g1 = wl, g0, g1
        self.seqs = [wl.sequence(b) for b in range(wl.cfg.B)]

    def __call__(self, q_local):
        cfg = self.wl.cfg
        G, scale32 = cfg.G, float(np.float32(1.0 / math.sqrt(cfg.d)))
        out = torch.zeros(cfg.B, (self.g1 - self.g0) * G, cfg.d, dtype=torch.float64)
        for b in range(cfg.B):
            keys, vals = self.seqs[b]
            L = cfg.lengths[b]
            for j, g in enumerate(range(self.g0, self.g1)):
                k = keys[g].float().numpy()
                v = vals[g].float().numpy()
                qg = q_local[b, j * G:(j + 1) * G].numpy()
                m = replica.page_meta(k, cfg.ps)
                _, ubg = replica.bound(qg, m["kmin"], m["kmax"], scale32)
                pages = select.topk(ubg, select.budget_pages(len(ubg), -1, 1 / 8))
                tok = attend.token_indices(pages, L, cfg.ps)
                o, _, _ = attend.entmax_attention(qg, k[tok], v[tok], cfg.alpha, 1.0 / math.sqrt(cfg.d))
                out[b, j * G:(j + 1) * G] = torch.from_numpy(o)
        return out


def _rank(rank, world, port, result):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = _workload()
        cfg = wl.cfg
        g0, g1 = kv_head_range(cfg.H_kv, world, rank)
        sharded = HeadShardedStep(OracleStep(wl, g0, g1), cfg.H_kv, cfg.G, world, rank)
        out = sharded(wl.q)
        result[rank] = out.numpy()
    finally:
        dist.destroy_process_group()


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_step_gathers_the_single_rank_output(world):
    with mp.get_context("spawn").Manager() as m:
        result = m.dict()
        mp.spawn(_rank, args=(world, _port(), result), nprocs=world, join=True)
        outs = [result[r] for r in range(world)]
    wl = _workload()
    ref = OracleStep(wl, 0, wl.cfg.H_kv)(wl.q).numpy()
    for r in range(world):
        assert np.array_equal(outs[r], ref), r              # every rank holds the whole output
