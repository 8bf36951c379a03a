"""Seeded synthetic workloads for the EntmaxKV decode step.

This module only draws inputs -- queries, keys, values, planted tokens,
sequence lengths and page tables -- with the shapes and distributions of the
five benchmark configurations.  It holds none of the method's arithmetic; the
tests feed the same tensors to the CUDA library and to the CPU oracle.

Recipes (every draw from a torch.Generator seeded per configuration and per
sequence, in a fixed order):

1 tiny:     B=1, 4 query / 1 kv heads, d=64, L=4096, ps=16, fp32 cache.
            Per-page centre c_p ~ N(0, I); key = c_p + 0.3 N(0, I).
            8 planted tokens, key = 3 q_h/|q_h| + 0.1 N(0, I).
2 llama:    B=1, 32/8 heads, d=128, L=131072, ps=64, bf16; same clustered
            keys; 64 planted tokens per kv head.
3 gauss:    B=4, 32/8, d=128, L=262144, ps=64, bf16.  Page centres follow a
            random walk c_0 ~ N(0, I), c_{p+1} = 0.9 c_p + 0.44 N(0, I); key =
            c_p + 0.5 N(0, I); per query head a log-uniform number in [16, 512]
            of planted tokens.
4 million:  B=1, 32/8, d=128, L=2^20, ps=64, bf16; clustered keys; 256
            planted tokens per kv head.
5 ragged:   B in {1, 8, 32}, 32/8, d=128, ps=64, bf16; L_b log-uniform in
            [32768, 524288]; clustered keys; physical pages a random
            permutation of one shared pool.

Planted tokens of a kv head are spread round-robin over its query heads; each
sits at a distinct uniformly drawn position.  Values ~ N(0, I); queries ~
N(0, I) fp32.  bf16 values are the round-to-nearest-even images of the fp32
draws.  Centres are drawn per (page, kv head).
"""
import math
from dataclasses import dataclass, field, replace
from typing import List

import torch


@dataclass
class Config:
    name: str
    B: int
    H_q: int
    H_kv: int
    d: int
    ps: int
    lengths: List[int]
    dtype: torch.dtype
    alpha: float = 1.5
    centres: str = "cluster"        # "cluster" or "walk"
    spread: float = 0.3
    planted_per_kv: int = 0         # cluster configs
    planted_range: tuple = ()       # walk config: (lo, hi) per query head, log-uniform
    budgets: List[int] = field(default_factory=list)      # pages
    budget_frac: float = -1.0
    deltas: List[float] = field(default_factory=list)
    alphas: List[float] = field(default_factory=list)
    permute_pages: bool = False
    decode_steps: int = 0
    seed: int = 1000

    @property
    def G(self):
        return self.H_q // self.H_kv

    @property
    def scale(self):
        return float(1.0 / math.sqrt(self.d))

    def pages(self, b):
        return (self.lengths[b] + self.ps - 1) // self.ps


def config(n, B=None, L=None):
    """Configuration n (1..5) of the benchmark suite; B and L override sizes."""
    if n == 1:
        c = Config("tiny", 1, 4, 1, 64, 16, [4096], torch.float32, planted_per_kv=8, budgets=[32], seed=1001)
    elif n == 2:
        c = Config("llama", 1, 32, 8, 128, 64, [131072], torch.bfloat16, planted_per_kv=64,
                   budgets=[64, 128, 256], seed=1002)
    elif n == 3:
        c = Config("gauss", 4, 32, 8, 128, 64, [262144] * 4, torch.bfloat16, centres="walk", spread=0.5,
                   planted_range=(16, 512), alphas=[1.5, 2.0], deltas=[0.0, 0.5, 1.0], seed=1003)
    elif n == 4:
        c = Config("million", 1, 32, 8, 128, 64, [1 << 20], torch.bfloat16, planted_per_kv=256,
                   budget_frac=1.0 / 64, deltas=[0.5], seed=1004)
    elif n == 5:
        Bn = 8 if B is None else B
        g = torch.Generator().manual_seed(1005)
        u = torch.rand(Bn, generator=g, dtype=torch.float64)
        lo, hi = math.log(32768), math.log(524288)
        lens = [int(round(math.exp(lo + (hi - lo) * float(x)))) for x in u]
        c = Config("ragged", Bn, 32, 8, 128, 64, lens, torch.bfloat16, planted_per_kv=64,
                   budget_frac=1.0 / 16, permute_pages=True, decode_steps=64, seed=1005)
    else:
        raise ValueError("configurations are numbered 1..5")
    if B is not None and n != 5:
        c = replace(c, B=B, lengths=[c.lengths[0]] * B)
    if L is not None:
        c = replace(c, lengths=[L] * c.B)
    return c


class Workload:
    """Deterministic inputs of one configuration on one device."""

    def __init__(self, cfg: Config, device="cpu", extra_pages=1):
        self.cfg = cfg
        self.device = torch.device(device)
        g = self._gen(0)
        self.q = torch.randn(cfg.B, cfg.H_q, cfg.d, generator=g, device=self.device, dtype=torch.float32)
        self.seq_lens_host = list(cfg.lengths)
        self.extra_pages = extra_pages + (cfg.decode_steps + cfg.ps - 1) // cfg.ps
        self.max_pages = max(cfg.pages(b) for b in range(cfg.B)) + self.extra_pages
        per_seq = [cfg.pages(b) + self.extra_pages for b in range(cfg.B)]
        self.num_phys = sum(per_seq)
        table = torch.zeros(cfg.B, self.max_pages, dtype=torch.int32)
        if cfg.permute_pages:
            perm = torch.randperm(self.num_phys, generator=torch.Generator().manual_seed(cfg.seed * 7 + 1))
        else:
            perm = torch.arange(self.num_phys)
        off = 0
        for b, n in enumerate(per_seq):
            table[b, :n] = perm[off:off + n].to(torch.int32)
            off += n
        self.page_table = table.to(self.device)

    def _gen(self, stream):
        seed = self.cfg.seed * 1_000_003 + stream
        return torch.Generator(device=self.device).manual_seed(seed)

    def seq_lens(self):
        return torch.tensor(self.seq_lens_host, dtype=torch.int32, device=self.device)

    def planted(self, b):
        """{query head: sorted token positions} of sequence b."""
        cfg = self.cfg
        L = cfg.lengths[b]
        g = torch.Generator().manual_seed(cfg.seed * 31 + b)
        heads = {}
        if cfg.planted_range:
            lo, hi = math.log(cfg.planted_range[0]), math.log(cfg.planted_range[1])
            counts = [int(round(math.exp(lo + (hi - lo) * float(torch.rand(1, generator=g, dtype=torch.float64)))))
                      for _ in range(cfg.H_q)]
        else:
            counts = []
            for kv in range(cfg.H_kv):
                for j in range(cfg.G):
                    counts.append(cfg.planted_per_kv // cfg.G + (1 if j < cfg.planted_per_kv % cfg.G else 0))
        for kv in range(cfg.H_kv):
            total = min(sum(counts[kv * cfg.G:(kv + 1) * cfg.G]), L)
            pos = torch.randperm(L, generator=g)[:total]
            # round-robin over the group's heads
            own = {h: [] for h in range(kv * cfg.G, (kv + 1) * cfg.G)}
            left = dict((h, counts[h]) for h in own)
            i = 0
            hs = sorted(own)
            while i < total:
                for h in hs:
                    if left[h] > 0 and i < total:
                        own[h].append(int(pos[i]))
                        left[h] -= 1
                        i += 1
            for h in hs:
                heads[h] = sorted(own[h])
        return heads

    def sequence(self, b, heads=None):
        """(keys, values) of sequence b, each [H_kv, L_b, d] in the cache dtype."""
        cfg = self.cfg
        L = cfg.lengths[b]
        P = cfg.pages(b)
        g = self._gen(1 + b)
        kvs = range(cfg.H_kv) if heads is None else heads
        keys, vals = [], []
        planted = self.planted(b)
        for kv in range(cfg.H_kv):
            # draw every head in order even when only some are returned
            if cfg.centres == "walk":
                c = torch.empty(P, cfg.d, device=self.device)
                c0 = torch.randn(cfg.d, generator=g, device=self.device)
                eps = torch.randn(P, cfg.d, generator=g, device=self.device)
                if P > 0:
                    c[0] = c0
                for p in range(1, P):
                    c[p] = 0.9 * c[p - 1] + 0.44 * eps[p]
            else:
                c = torch.randn(P, cfg.d, generator=g, device=self.device)
            k = torch.randn(L, cfg.d, generator=g, device=self.device)
            k.mul_(cfg.spread).add_(c.repeat_interleave(cfg.ps, dim=0)[:L])
            for h in range(kv * cfg.G, (kv + 1) * cfg.G):
                pos = planted[h]
                if pos:
                    qh = self.q[b, h]
                    noise = torch.randn(len(pos), cfg.d, generator=g, device=self.device)
                    k[torch.tensor(pos, device=self.device)] = 3.0 * qh / qh.norm() + 0.1 * noise
            v = torch.randn(L, cfg.d, generator=g, device=self.device)
            if kv in kvs:
                keys.append(k.to(cfg.dtype))
                vals.append(v.to(cfg.dtype))
            del k, v, c
        return torch.stack(keys), torch.stack(vals)

    def decode_token(self, step):
        """(k, v) [B, H_kv, 1, d] appended at decode step `step`, and the step's query."""
        cfg = self.cfg
        g = self._gen(100_000 + step)
        k = torch.randn(cfg.B, cfg.H_kv, 1, cfg.d, generator=g, device=self.device).to(cfg.dtype)
        v = torch.randn(cfg.B, cfg.H_kv, 1, cfg.d, generator=g, device=self.device).to(cfg.dtype)
        q = torch.randn(cfg.B, cfg.H_q, cfg.d, generator=g, device=self.device)
        return k, v, q
