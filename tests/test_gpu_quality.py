"""Sparse softmax decoding at a matched budget, and the entmax-versus-softmax
comparison of the EntmaxKV pages on the synthetic generators.

German technical summary, section 3: the output error of decoding over a kept
subset is bounded by 2 B delta (B bounds the value norms, delta is the full-cache
probability mass of the dropped tokens); softmax has delta > 0 as soon as any
token is dropped, alpha-entmax has delta = 0 whenever the kept set contains the
support.  Section 4: at matched KV budgets entmax drops less mass, keeps more of
the support and has a lower relative output error.

Every output here comes from the CUDA library through the C ABI; delta and the
support recall come from the oracle's full-cache probabilities.
"""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

import helpers as H
from oracle import attend, entmax, select
from sparse_long_context_min_b200 import binding as B
from sparse_long_context_min_b200 import workloads
from sparse_long_context_min_b200.step import DecodeStep, build_pool

pytestmark = pytest.mark.gpu


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _ok(st):
    torch.cuda.synchronize()
    assert int(st.item()) == 0, B.status_string(int(st.item()))


def _wl(n, L):
    cfg = replace(workloads.config(n), B=1, lengths=[L])
    return workloads.Workload(cfg, device="cuda")


def _softmax_ws(cfg, max_pages, k_max):
    n = B.workspace_size(B.OP_SPARSE_SOFTMAX, cfg.B, cfg.H_q, cfg.H_kv, max_pages, k_max, cfg.ps, cfg.d)
    return torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("n,L", [(1, 4096 + 5), (2, 16384 + 1)])
def test_sparse_softmax_against_oracle(n, L):
    """GPU softmax over a given page list equals the oracle's softmax over the
    valid tokens of those pages (an empty list gives zeros)."""
    wl = _wl(n, L)
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    o = H.OracleSeq(wl, 0)
    P = cfg.pages(0)
    k_max = max(1, math.ceil(P / 8))
    sel = torch.zeros(1, cfg.H_kv, k_max, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, cfg.H_kv, dtype=torch.int32, device="cuda")
    lists = {}
    for g in range(cfg.H_kv):
        if g == cfg.H_kv - 1 and cfg.H_kv > 1:
            pages = np.zeros(0, dtype=np.int64)                    # empty list
        else:
            pages = o.topk(g, -1, 1 / 8)
            if P - 1 not in set(pages.tolist()):                   # include the ragged last page
                pages = np.array(sorted(set(pages.tolist()[1:]) | {P - 1}))
        sel[0, g, :len(pages)] = torch.from_numpy(pages.astype(np.int32))
        cnt[0, g] = len(pages)
        lists[g] = pages
    out = torch.full((1, cfg.H_q, cfg.d), 7.0, device="cuda")
    st = _status()
    B.sparse_softmax_attend(pool, wl.q, wl.page_table, seq_lens, sel, cnt, H.scale32(cfg), out,
                            _softmax_ws(cfg, wl.max_pages, k_max), st)
    _ok(st)
    out = out.cpu().numpy()
    G = cfg.G
    for g, pages in lists.items():
        got = out[0, g * G:(g + 1) * G]
        if len(pages) == 0:
            assert np.all(got == 0.0)
            continue
        tok = attend.token_indices(pages, o.L, cfg.ps)
        ref = attend.softmax_attention(o.qgroup(g), o.keys[g][tok], o.values[g][tok], 1 / math.sqrt(cfg.d))
        H.compare_out(got, ref, cfg.dtype)


def test_sparse_softmax_with_every_page_equals_full_softmax():
    wl = _wl(2, 9000)
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    P = cfg.pages(0)
    sel = torch.arange(P, dtype=torch.int32, device="cuda").repeat(1, cfg.H_kv, 1).contiguous()
    cnt = torch.full((1, cfg.H_kv), P, dtype=torch.int32, device="cuda")
    a = torch.empty(1, cfg.H_q, cfg.d, device="cuda")
    b = torch.empty_like(a)
    st = _status()
    B.sparse_softmax_attend(pool, wl.q, wl.page_table, seq_lens, sel, cnt, H.scale32(cfg), a,
                            _softmax_ws(cfg, wl.max_pages, P), st)
    ws = torch.empty(B.workspace_size(B.OP_FULL_SOFTMAX, 1, cfg.H_q, cfg.H_kv, wl.max_pages, 0, cfg.ps, cfg.d),
                     dtype=torch.uint8, device="cuda")
    B.full_softmax_decode(pool, wl.q, wl.page_table, seq_lens, H.scale32(cfg), b, ws, st)
    _ok(st)
    assert torch.allclose(a, b, rtol=0, atol=1e-5)


BUDGETS = (1 / 64, 1 / 16, 1 / 4, 1 / 2, 1.0)


def test_matched_budget_entmax_versus_softmax(capsys):
    """Top-k selections at several budgets; sparse entmax and sparse softmax on
    the same kept set against their full-cache outputs.  Checks what the pages
    state as facts (error bound, softmax's dense tail, exactness once the support
    is kept) and prints the sweep (delta, recall, relative error)."""
    wl = _wl(2, 16384 + 1)
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    o = H.OracleSeq(wl, 0)
    P = cfg.pages(0)
    G, d = cfg.G, cfg.d
    scale = H.scale32(cfg)
    st = _status()
    # full-cache references (GPU)
    full_e = torch.empty(1, cfg.H_q, d, device="cuda")
    full_s = torch.empty_like(full_e)
    ws_e = torch.empty(B.workspace_size(B.OP_FULL_ENTMAX, 1, cfg.H_q, cfg.H_kv, wl.max_pages, 0, cfg.ps, d),
                       dtype=torch.uint8, device="cuda")
    ws_s = torch.empty(B.workspace_size(B.OP_FULL_SOFTMAX, 1, cfg.H_q, cfg.H_kv, wl.max_pages, 0, cfg.ps, d),
                       dtype=torch.uint8, device="cuda")
    B.full_entmax_decode(pool, wl.q, wl.page_table, seq_lens, cfg.alpha, scale, full_e, ws_e, st)
    B.full_softmax_decode(pool, wl.q, wl.page_table, seq_lens, scale, full_s, ws_s, st)
    _ok(st)
    full_e, full_s = full_e.cpu().numpy()[0], full_s.cpu().numpy()[0]
    # oracle full-cache probabilities of two kv heads' query heads
    heads = (0, 5)
    pe, ps_ = {}, {}
    for g in heads:
        x_scores = (1 / math.sqrt(d)) * np.stack([(o.keys[g].astype(np.float64) * o.qgroup(g)[h]).sum(axis=1)
                                                  for h in range(G)])
        pe[g] = np.stack([entmax.probs((cfg.alpha - 1) * x_scores[h], cfg.alpha)[0] for h in range(G)])
        ps_[g] = np.stack([entmax.softmax(x_scores[h]) for h in range(G)])
    vnorm = float(np.linalg.norm(o.values.astype(np.float64), axis=-1).max())
    tol = 0.03                                    # norm over d of bf16-path output errors
    rows = []
    for frac in BUDGETS:
        step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=frac, alpha=cfg.alpha)
        step.score(wl.q)
        step.choose()
        step.attend(wl.q)
        out_s = torch.empty_like(step.out)
        B.sparse_softmax_attend(pool, wl.q, wl.page_table, seq_lens, step.sel, step.sel_count, scale, out_s,
                                _softmax_ws(cfg, wl.max_pages, step.k_max), step.status)
        step.check()
        sel, cnt = step.sel.cpu().numpy(), step.sel_count.cpu().numpy()
        out_e, out_s = step.out.cpu().numpy()[0], out_s.cpu().numpy()[0]
        for g in heads:
            pages = sel[0, g, :cnt[0, g]]
            assert np.array_equal(pages, o.topk(g, -1, frac))
            tok = attend.token_indices(pages, o.L, cfg.ps)
            de = attend.dropped_mass(pe[g], tok)
            ds = attend.dropped_mass(ps_[g], tok)
            rec = attend.support_recall(pe[g], tok)
            sl = slice(g * G, (g + 1) * G)
            ee = np.linalg.norm(out_e[sl] - full_e[sl], axis=1)
            es = np.linalg.norm(out_s[sl] - full_s[sl], axis=1)
            # section 3: ||o - o~|| <= 2 B delta, for both distributions
            assert np.all(ee <= 2 * vnorm * de + tol), (frac, g, ee, de)
            assert np.all(es <= 2 * vnorm * ds + tol), (frac, g, es, ds)
            if len(pages) < P:
                assert np.all(ds > 0)                 # softmax's dense tail
            else:
                assert np.all(de == 0) and np.all(ds == 0)
            kept_support = rec == 1.0
            assert np.all(de[kept_support] == 0)
            assert np.all(ee[kept_support] <= tol)    # exact once the support is kept
            ne = np.linalg.norm(full_e[sl], axis=1)
            ns = np.linalg.norm(full_s[sl], axis=1)
            rows.append((frac, len(pages), de.mean(), ds.mean(), rec.mean(), (ee / ne).mean(), (es / ns).mean()))
    with capsys.disabled():
        print("\nbudget  pages  delta_entmax  delta_softmax  recall  relerr_entmax  relerr_softmax")
        for r in rows:
            print("%6.4f %6d %13.4f %14.4f %7.3f %14.4f %15.4f" % r)
