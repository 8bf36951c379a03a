"""The two selectors against context length (German summary, section 4: the
Gaussian-aware selector adapts its budget to the score distribution instead of
a fixed top-k).

Configuration 4's generator (B = 1, 32/8 heads, d = 128, pages of 64, bf16,
clustered keys with 256 planted tokens per kv head) at 2^18, 2^19 and 2^20
tokens.  For top-k 1/64 and the Gaussian selector with Delta = 0.5, on sampled
kv heads: the selection (top-k against the replica bounds, the Gaussian keep
rule against the replica estimates at the GPU's tau_hat), the attention output
against the oracle on the kept set, and the dropped mass delta and support
recall from the oracle's full-cache probabilities (delta = 0 wherever the
support is kept).  One line per (length, selector) is printed; bench.py
--selector-sweep times the same steps.
"""
import math
from dataclasses import replace

import numpy as np
import pytest

import helpers as H
from oracle import attend, replica, select
from sparse_long_context_min_b200 import workloads
from sparse_long_context_min_b200.step import DecodeStep, build_pool

pytestmark = pytest.mark.gpu

HEADS = (1, 6)


@pytest.mark.parametrize("L", [1 << 18, 1 << 19, 1 << 20])
def test_selectors_against_length(L, capsys):
    cfg = replace(workloads.config(4), lengths=[L])
    wl = workloads.Workload(cfg, device="cuda")
    pool, seq_lens = build_pool(wl)
    G, scale = cfg.G, 1.0 / math.sqrt(cfg.d)
    q = wl.q[0].cpu().numpy()
    rows = []
    steps = {}
    for mode in ("topk", "gauss"):
        st = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, mode, budget_frac=1 / 64, alpha=cfg.alpha, delta=0.5)
        st(wl.q)
        st.check()
        steps[mode] = (st.sel.cpu().numpy(), st.sel_count.cpu().numpy(), st.out.cpu().numpy(),
                       None if st.tau_hat is None else st.tau_hat.cpu().numpy())
    for g in HEADS:
        keys, vals = wl.sequence(0, heads=[g])
        k, v = keys[0].float().cpu().numpy(), vals[0].float().cpu().numpy()
        meta = replica.page_meta(k, cfg.ps)
        qg = q[g * G:(g + 1) * G]
        _, _, p_full = attend.entmax_attention(qg, k, v, cfg.alpha, scale)
        for mode, (sel, cnt, out, tau_hat) in steps.items():
            kept = sel[0, g, :cnt[0, g]]
            if mode == "topk":
                _, ubg = replica.bound(qg, meta["kmin"], meta["kmax"], H.scale32(cfg))
                assert np.array_equal(kept, select.topk(ubg, select.budget_pages(len(ubg), -1, 1 / 64)))
            else:
                _, _, est = replica.gauss(qg, meta["mean"], meta["m2"], meta["count"], H.scale32(cfg), cfg.ps)
                assert np.array_equal(kept, select.gauss_keep(est, tau_hat[0, g * G:(g + 1) * G], cfg.alpha, 0.5))
            tok = attend.token_indices(kept, L, cfg.ps)
            o_ref, _, _ = attend.entmax_attention(qg, k[tok], v[tok], cfg.alpha, scale)
            H.compare_out(out[0, g * G:(g + 1) * G], o_ref, cfg.dtype)
            dm = attend.dropped_mass(p_full, tok)
            rec = attend.support_recall(p_full, tok)
            assert np.all(dm[rec == 1.0] == 0.0)
            rows.append((mode, g, len(kept), float(dm.mean()), float(dm.max()), float(rec.mean())))
    with capsys.disabled():
        P = cfg.pages(0)
        for mode in ("topk", "gauss"):
            r = [x for x in rows if x[0] == mode]
            print("\nselector %-5s L=%7d: pages kept per kv head %s of %d; delta mean %.3g max %.3g; recall mean %.4f"
                  % (mode, L, "/".join(str(x[2]) for x in r), P, np.mean([x[3] for x in r]),
                     max(x[4] for x in r), np.mean([x[5] for x in r])))
