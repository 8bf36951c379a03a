"""Configuration 3 at full size: the Gaussian-aware selector's budget and its
dropped mass.

B = 4 sequences of 262144 tokens, 32 query / 8 kv heads, d = 128, pages of 64,
bf16 cache, random-walk page centres with a planted support of 16-512 tokens
per query head; alpha in {1.5, 2}, Delta in {0, 0.5, 1}.  For every (alpha,
Delta) the configuration names, the decode step (Gaussian scoring, tau_hat,
keep rule, sparse entmax attention) runs on the GPU through the C ABI, and:

* every (sequence, kv head): the kept set equals, bit for bit, the fp32 keep
  rule evaluated with the GPU's own tau_hat on the replica's page estimates;
* sampled (sequence, kv head) pairs: tau_hat within its tolerance of the
  oracle's float64 root; the attention output against the oracle fed the GPU's
  kept set; the dropped mass delta and the support recall from the oracle's
  full-cache probabilities, with the facts of the German technical summary,
  section 3: delta = 0 whenever the kept pages hold the support, and
  ||o_sparse - o_full|| <= 2 B delta (B the largest value norm);
* the selected budget (pages kept per kv head), delta and recall are printed
  as one table row per (alpha, Delta).
"""
import math

import numpy as np
import pytest
import torch

import helpers as H
from oracle import attend, entmax, gauss, replica, select
from sparse_long_context_min_b200 import workloads
from sparse_long_context_min_b200.step import DecodeStep, build_pool

pytestmark = pytest.mark.gpu

SAMPLES = [(0, 3), (1, 0), (2, 5), (3, 7)]
TOL = 0.03          # norm over d of the bf16 path's output error (as in the quality sweep)


class Config3:
    """The configuration-3 pool on the GPU plus oracle-side data that does not
    depend on alpha or Delta: page metadata of every (sequence, kv head), and
    keys and values of the sampled pairs."""

    def __init__(self):
        self.wl = workloads.Workload(workloads.config(3), device="cuda")
        self.cfg = self.wl.cfg
        self.pool, self.seq_lens = build_pool(self.wl)
        self.meta, self.kv = {}, {}
        for b in range(self.cfg.B):
            keys, vals = self.wl.sequence(b)
            for g in range(self.cfg.H_kv):
                k = keys[g].float().cpu().numpy()
                self.meta[b, g] = replica.page_meta(k, self.cfg.ps)
                if (b, g) in SAMPLES:
                    self.kv[b, g] = (k, vals[g].float().cpu().numpy())
            del keys, vals
            torch.cuda.empty_cache()
        self.q = self.wl.q.cpu().numpy()
        self._pfull = {}

    def qgroup(self, b, g):
        G = self.cfg.G
        return self.q[b, g * G:(g + 1) * G]

    def est(self, b, g):
        m = self.meta[b, g]
        return replica.gauss(self.qgroup(b, g), m["mean"], m["m2"], m["count"], H.scale32(self.cfg), self.cfg.ps)

    def p_full(self, b, g, alpha):
        """Full-cache alpha-entmax probabilities [G, L] and output [G, d] (float64)."""
        key = (b, g, alpha)
        if key not in self._pfull:
            k, v = self.kv[b, g]
            o, _, p = attend.entmax_attention(self.qgroup(b, g), k, v, alpha, 1.0 / math.sqrt(self.cfg.d))
            self._pfull[key] = (p, o)
        return self._pfull[key]


@pytest.fixture(scope="module")
def c3():
    return Config3()


@pytest.mark.parametrize("alpha", [1.5, 2.0])
@pytest.mark.parametrize("delta", [0.0, 0.5, 1.0])
def test_config3_budget_and_dropped_mass(c3, alpha, delta, capsys):
    cfg, wl = c3.cfg, c3.wl
    G, P = cfg.G, cfg.pages(0)
    step = DecodeStep(c3.pool, wl.page_table, c3.seq_lens, cfg.H_q, "gauss", alpha=alpha, delta=delta)
    step(wl.q)
    step.check()
    sel, cnt = step.sel.cpu().numpy(), step.sel_count.cpu().numpy()
    tau_gpu, out = step.tau_hat.cpu().numpy(), step.out.cpu().numpy()
    for b in range(cfg.B):
        for g in range(cfg.H_kv):
            _, _, est = c3.est(b, g)
            kept = sel[b, g, :cnt[b, g]]
            assert np.array_equal(kept, select.gauss_keep(est, tau_gpu[b, g * G:(g + 1) * G], alpha, delta)), \
                (b, g)
    deltas, recalls = [], []
    for b, g in SAMPLES:
        m, v, est = c3.est(b, g)
        n = c3.meta[b, g]["count"]
        ref = np.array([gauss.tau_hat(m[h].astype(np.float64), v[h].astype(np.float64), n, alpha)
                        for h in range(G)])
        got = tau_gpu[b, g * G:(g + 1) * G].astype(np.float64)
        assert np.all(np.abs(got - ref) <= H.TAU_HAT_TOL * np.maximum(1.0, np.abs(ref))), (got, ref)
        k, vals = c3.kv[b, g]
        kept = sel[b, g, :cnt[b, g]]
        tok = attend.token_indices(kept, cfg.lengths[b], cfg.ps)
        o_ref, _, _ = attend.entmax_attention(c3.qgroup(b, g), k[tok], vals[tok], alpha, 1.0 / math.sqrt(cfg.d))
        o_gpu = out[b, g * G:(g + 1) * G]
        H.compare_out(o_gpu, o_ref, cfg.dtype)
        p_full, o_full = c3.p_full(b, g, alpha)
        dm = attend.dropped_mass(p_full, tok)
        rec = attend.support_recall(p_full, tok)
        assert np.all(dm[rec == 1.0] == 0.0)
        vnorm = float(np.linalg.norm(vals.astype(np.float64), axis=1).max())
        err = np.linalg.norm(o_gpu.astype(np.float64) - o_full, axis=1)
        assert np.all(err <= 2.0 * vnorm * dm + TOL), (err, dm)
        deltas.extend(dm.tolist())
        recalls.extend(rec.tolist())
    kept_pages = cnt.astype(np.float64)
    with capsys.disabled():
        print("\nconfig3 alpha=%.1f Delta=%.1f: pages kept per kv head mean %.1f (min %d, max %d) of %d = %.4f; "
              "sampled query heads: delta mean %.3g max %.3g, recall mean %.4f, heads with recall 1: %d/%d"
              % (alpha, delta, kept_pages.mean(), int(cnt.min()), int(cnt.max()), P, kept_pages.mean() / P,
                 float(np.mean(deltas)), float(np.max(deltas)), float(np.mean(recalls)),
                 int(np.sum(np.asarray(recalls) == 1.0)), len(recalls)))
