"""Shared helpers of the GPU parity tests: oracle-side views of a workload.

The oracle side is always computed from the generator's tensors (copied to the
host), never from anything the CUDA library wrote.
"""
import math

import numpy as np
import torch

from oracle import attend, gauss, replica, select
from sparse_long_context_min_b200 import workloads

BF16_ATOL = 2e-3      # absolute, bf16 cache with fp32 accumulation
F32_RTOL = 1e-5       # relative to the head's largest |o|, fp32 cache
TAU_HAT_TOL = 1e-4    # relative to max(1, |tau_hat|)


def host_sequence(wl, b):
    """(keys, values) of sequence b as float32 numpy [H_kv, L, d] (bf16 widened exactly)."""
    k, v = wl.sequence(b)
    return k.float().cpu().numpy(), v.float().cpu().numpy()


def scale32(cfg):
    return float(np.float32(1.0 / math.sqrt(cfg.d)))


class OracleSeq:
    """Oracle metadata and scores of one sequence, per kv head (lazily)."""

    def __init__(self, wl, b):
        self.wl, self.b, self.cfg = wl, b, wl.cfg
        self.keys, self.values = host_sequence(wl, b)
        self.q = wl.q[b].float().cpu().numpy()
        self.L = self.cfg.lengths[b]
        self._meta = {}

    def meta(self, g):
        if g not in self._meta:
            self._meta[g] = replica.page_meta(self.keys[g], self.cfg.ps)
        return self._meta[g]

    def qgroup(self, g):
        G = self.cfg.G
        return self.q[g * G:(g + 1) * G]

    def ubg(self, g):
        m = self.meta(g)
        return replica.bound(self.qgroup(g), m["kmin"], m["kmax"], scale32(self.cfg))[1]

    def gauss(self, g):
        m = self.meta(g)
        return replica.gauss(self.qgroup(g), m["mean"], m["m2"], m["count"], scale32(self.cfg), self.cfg.ps)

    def topk(self, g, budget=-1, frac=0.0):
        P = (self.L + self.cfg.ps - 1) // self.cfg.ps
        k = select.budget_pages(P, budget, frac)
        return select.topk(self.ubg(g), k)

    def attention(self, g, pages, alpha):
        tok = attend.token_indices(pages, self.L, self.cfg.ps)
        o, tau, _ = attend.entmax_attention(self.qgroup(g), self.keys[g][tok], self.values[g][tok], alpha,
                                            1.0 / math.sqrt(self.cfg.d))
        return o, tau

    def tau_hat(self, g, alpha):
        m, v, _ = self.gauss(g)
        n = self.meta(g)["count"]
        return np.array([gauss.tau_hat(m[h].astype(np.float64), v[h].astype(np.float64), n, alpha)
                         for h in range(self.cfg.G)])


def compare_out(o_gpu, o_ref, dtype):
    """Assert the attention output tolerance of the cache dtype; return the error."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    if dtype == torch.float32:
        err = np.abs(o_gpu - o_ref).max(axis=-1) / np.maximum(np.abs(o_ref).max(axis=-1), 1e-30)
        assert err.max() <= F32_RTOL, err.max()
    else:
        err = np.abs(o_gpu - o_ref).max()
        assert err <= BF16_ATOL, err
    return float(np.max(err))


def small_config(n, **kw):
    return workloads.config(n, **kw)
