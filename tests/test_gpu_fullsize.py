"""GPU parity at the benchmark configurations' full sizes, on sampled heads.

Every configuration runs at its stated size through the path bench.py times
(the step captured as one CUDA graph: append, score, select, attend).  The
oracle recomputes, for a few sampled (sequence, kv head) pairs, the page
metadata from the generated keys (including the appended decode tokens), the
selection, and the entmax attention of the group's query heads.
"""
import math

import numpy as np
import pytest

import helpers as H
from oracle import attend, gauss, replica, select
from sparse_long_context_min_b200 import workloads
from sparse_long_context_min_b200.step import DecodeStep, GraphedStep, build_pool

pytestmark = pytest.mark.gpu


def _graphed_steps(wl, pool, seq_lens, mode, n_steps, **kw):
    cfg = wl.cfg
    st = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, mode, alpha=kw.pop("alpha", cfg.alpha), **kw)
    gs = GraphedStep(st, append=True, stage_events=False)
    toks = []
    for t in range(n_steps):
        k, v, q = wl.decode_token(t)
        gs.q.copy_(q)
        gs.k.copy_(k)
        gs.v.copy_(v)
        gs.replay()
        toks.append((k, v, q))
    st.check()
    return st, toks


def _oracle_seq(wl, b, toks):
    """(keys, values) [H_kv, L + appended, d] float32 of sequence b, last query."""
    keys, vals = H.host_sequence(wl, b)
    if toks:
        keys = np.concatenate([keys] + [t[0][b].float().cpu().numpy() for t in toks], axis=1)
        vals = np.concatenate([vals] + [t[1][b].float().cpu().numpy() for t in toks], axis=1)
    return keys, vals, toks[-1][2][b].float().cpu().numpy()


def _check_topk(wl, st, toks, samples, frac=None, budget=-1, select_all=False):
    """Top-k sets against the replica bounds (every kv head of every sequence
    when select_all, else the sampled ones) and the entmax attention of the
    sampled (sequence, kv head) pairs against the oracle."""
    cfg = wl.cfg
    G = cfg.G
    sel, cnt, out = st.sel.cpu().numpy(), st.sel_count.cpu().numpy(), st.out.cpu().numpy()
    heads = [(b, g) for b in range(cfg.B) for g in range(cfg.H_kv)] if select_all else list(samples)
    seqs = {}
    for b, g in heads:
        if b not in seqs:
            seqs[b] = _oracle_seq(wl, b, toks)
        keys, vals, q = seqs[b]
        L = keys.shape[1]
        meta = replica.page_meta(keys[g], cfg.ps)
        qg = q[g * G:(g + 1) * G]
        _, ubg = replica.bound(qg, meta["kmin"], meta["kmax"], H.scale32(cfg))
        pages = select.topk(ubg, select.budget_pages(len(ubg), budget, frac if frac is not None else 0.0))
        assert np.array_equal(sel[b, g, :cnt[b, g]], pages), (b, g)
        if (b, g) not in samples:
            continue
        tok = attend.token_indices(pages, L, cfg.ps)
        o_ref, _, _ = attend.entmax_attention(qg, keys[g][tok], vals[g][tok], cfg.alpha, 1 / math.sqrt(cfg.d))
        H.compare_out(out[b, g * G:(g + 1) * G], o_ref, cfg.dtype)


def test_config1_tiny_all_heads():
    wl = workloads.Workload(workloads.config(1), device="cuda")
    pool, seq_lens = build_pool(wl)
    st, toks = _graphed_steps(wl, pool, seq_lens, "topk", 2, budget=32)
    _check_topk(wl, st, toks, [(0, 0)], budget=32)


@pytest.mark.parametrize("budget", [64, 128, 256])
def test_config2_llama_budgets(budget):
    wl = workloads.Workload(workloads.config(2), device="cuda")
    pool, seq_lens = build_pool(wl)
    st, toks = _graphed_steps(wl, pool, seq_lens, "topk", 2, budget=budget)
    _check_topk(wl, st, toks, [(0, 1), (0, 6)], budget=budget, select_all=True)


def test_config4_million_topk():
    wl = workloads.Workload(workloads.config(4), device="cuda")
    pool, seq_lens = build_pool(wl)
    st, toks = _graphed_steps(wl, pool, seq_lens, "topk", 3, budget_frac=1 / 64)
    _check_topk(wl, st, toks, [(0, 0), (0, 5)], frac=1 / 64, select_all=True)


def _check_gauss(wl, st, toks, samples, alpha, delta):
    """Gaussian selection of the sampled (sequence, kv head) pairs: tau_hat
    within its tolerance of the oracle's float64 root, the kept set equal bit
    for bit to the fp32 keep rule at the GPU's own threshold (decisions against
    the oracle's threshold may differ only inside the band its error spans),
    and the attention output against the oracle fed the GPU's kept set."""
    cfg = wl.cfg
    G = cfg.G
    sel, cnt, out = st.sel.cpu().numpy(), st.sel_count.cpu().numpy(), st.out.cpu().numpy()
    tau_gpu = st.tau_hat.cpu().numpy()
    for b, g in samples:
        keys, vals, q = _oracle_seq(wl, b, toks)
        L = keys.shape[1]
        meta = replica.page_meta(keys[g], cfg.ps)
        qg = q[g * G:(g + 1) * G]
        m, v, est = replica.gauss(qg, meta["mean"], meta["m2"], meta["count"], H.scale32(cfg), cfg.ps)
        ref = np.array([gauss.tau_hat(m[h].astype(np.float64), v[h].astype(np.float64), meta["count"], alpha)
                        for h in range(G)])
        got = tau_gpu[b, g * G:(g + 1) * G]
        g64 = got.astype(np.float64)
        assert np.all(np.abs(g64 - ref) <= H.TAU_HAT_TOL * np.maximum(1.0, np.abs(ref))), (got, ref)
        kept = sel[b, g, :cnt[b, g]]
        assert np.array_equal(kept, select.gauss_keep(est, got, alpha, delta)), (b, g)
        band = np.abs(g64 - ref) + 1e-6 * np.maximum(1.0, np.abs(ref))
        must_keep, must_drop = select.gauss_keep_bands(est, ref, alpha, delta, band[:, None])
        own = select.gauss_keep(est, ref.astype(np.float32), alpha, delta)
        diff = set(own.tolist()) ^ set(kept.tolist())
        assert not (diff & (set(must_keep.tolist()) | set(must_drop.tolist())))
        tok = attend.token_indices(kept, L, cfg.ps)
        o_ref, _, _ = attend.entmax_attention(qg, keys[g][tok], vals[g][tok], alpha, 1 / math.sqrt(cfg.d))
        H.compare_out(out[b, g * G:(g + 1) * G], o_ref, cfg.dtype)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
@pytest.mark.parametrize("delta", [0.0, 0.5, 1.0])
def test_config3_gauss_full(alpha, delta):
    wl = workloads.Workload(workloads.config(3), device="cuda")
    pool, seq_lens = build_pool(wl)
    st, toks = _graphed_steps(wl, pool, seq_lens, "gauss", 1, alpha=alpha, delta=delta)
    _check_gauss(wl, st, toks, [(0, 3), (3, 7)], alpha, delta)


def test_config4_million_gauss():
    wl = workloads.Workload(workloads.config(4), device="cuda")
    pool, seq_lens = build_pool(wl)
    st, toks = _graphed_steps(wl, pool, seq_lens, "gauss", 1, delta=0.5)
    _check_gauss(wl, st, toks, [(0, 2)], 1.5, 0.5)


@pytest.mark.parametrize("B", [1, 8, 32])
def test_config5_ragged_64_decode_steps(B):
    wl = workloads.Workload(workloads.config(5, B=B), device="cuda")
    pool, seq_lens = build_pool(wl)
    st, toks = _graphed_steps(wl, pool, seq_lens, "topk", 64, budget_frac=1 / 16)
    assert seq_lens.cpu().tolist() == [L + 64 for L in wl.cfg.lengths]
    _check_topk(wl, st, toks, [(0, 0), (B - 1, 4)], frac=1 / 16)
