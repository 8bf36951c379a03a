"""Pins of the page-metadata and page-score oracle (c2, c3) and its fp32 replicas.

* worked examples (box bound, Welford) from tests/golden;
* the bound is >= every true score in its page (the defining property) and is
  attained when a key sits on the maximising corner;
* a single-token page has kmin = kmax = k, so its bound equals the exact score;
* the f64 moments satisfy var = E[k^2] - E[k]^2 and translation invariance;
* the fp32 replicas agree with the f64 definitions within fp32 rounding, the
  replica's kmin/kmax equal the exact minima/maxima, and an incrementally built
  page equals a whole-page build bit for bit.
"""
import json
import os

import numpy as np
import pytest

from oracle import gauss, pages, replica

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def _bf16_round(a):
    """Round fp32 to bf16 (nearest-even) and widen back, in numpy."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _keys(rng, L, d, ps, spread=0.3):
    P = (L + ps - 1) // ps
    c = rng.standard_normal((P, d))
    k = np.repeat(c, ps, axis=0)[:L] + spread * rng.standard_normal((L, d))
    return _bf16_round(k)


def test_golden_bbox_and_welford():
    ex = GOLD["bbox"][0]
    q = np.array([ex["q"]])
    ub = pages.bbox_bound(q, np.array([ex["kmin"]]), np.array([ex["kmax"]]), ex["scale"])
    assert ub[0, 0] == ex["ub"]
    assert float(q[0] @ np.array(ex["corner_key"])) == ex["ub"]
    # the fp32 replica works on d a multiple of 8: zero coordinates add nothing
    pad = lambda a: np.pad(np.asarray(a, dtype=float), ((0, 0), (0, 6)))  # noqa: E731
    _, ubg = replica.bound(pad(q), pad([ex["kmin"]]), pad([ex["kmax"]]), ex["scale"])
    assert ubg[0] == np.float32(ex["ub"])
    w = GOLD["welford"][0]
    tok = np.array(w["tokens"])[:, None]
    meta = pages.page_metadata(tok, ps=4)
    assert abs(meta["mean"][0, 0] - w["mean"]) < 1e-15
    assert abs(meta["var"][0, 0] - w["var"]) < 1e-15
    rm = replica.page_meta(tok, ps=4)
    assert abs(rm["mean"][0, 0] - w["mean"]) < 1e-6
    assert abs(rm["m2"][0, 0] / 3.0 - w["var"]) < 1e-6


@pytest.mark.parametrize("ps,d", [(16, 64), (64, 128)])
def test_bound_dominates_every_score(ps, d):
    rng = np.random.default_rng(10)
    L = 7 * ps + 5          # ragged last page
    keys = _keys(rng, L, d, ps)
    q = rng.standard_normal((4, d)).astype(np.float32)
    scale = 1.0 / np.sqrt(d)
    meta = pages.page_metadata(keys, ps)
    ub = pages.bbox_bound(q, meta["kmin"], meta["kmax"], scale)
    true = pages.true_page_max(q, keys, ps, scale)
    assert ub.shape == true.shape == (4, 8)
    assert (ub >= true - 1e-12).all()
    # fp32 replica: same bound up to fp32 rounding of a d-term sum
    _, ubg = replica.bound(q, meta["kmin"], meta["kmax"], scale)
    np.testing.assert_allclose(ubg, ub.max(axis=0), rtol=1e-5, atol=1e-5)
    assert (ubg.astype(np.float64) >= true.max(axis=0) - 1e-4).all()


def test_bound_of_single_token_page_is_exact():
    rng = np.random.default_rng(11)
    d = 64
    keys = _keys(rng, 9, d, 1)
    q = rng.standard_normal((3, d))
    meta = pages.page_metadata(keys, 1)
    ub = pages.bbox_bound(q, meta["kmin"], meta["kmax"], 0.125)
    np.testing.assert_allclose(ub, 0.125 * q @ keys.T, rtol=1e-13, atol=1e-13)
    ubr, _ = replica.bound(q.astype(np.float32), meta["kmin"], meta["kmax"], 0.125)
    np.testing.assert_allclose(ubr, 0.125 * q.astype(np.float32) @ keys.T, rtol=1e-5, atol=1e-5)


def test_bound_attained_on_corner():
    rng = np.random.default_rng(12)
    d = 32
    q = rng.standard_normal((1, d))
    keys = rng.standard_normal((16, d))
    kmin, kmax = keys.min(0), keys.max(0)
    corner = np.where(q[0] >= 0, kmax, kmin)
    keys = np.vstack([keys, corner])
    meta = pages.page_metadata(keys, 17)
    ub = pages.bbox_bound(q, meta["kmin"], meta["kmax"], 1.0)
    assert abs(ub[0, 0] - q[0] @ corner) < 1e-12


def test_moments_invariants():
    rng = np.random.default_rng(13)
    keys = rng.standard_normal((100, 8)) * 3 + 1
    meta = pages.page_metadata(keys, 32)
    for p in range(4):
        blk = keys[p * 32:(p + 1) * 32]
        ex2 = (blk ** 2).sum(0) / blk.shape[0]
        np.testing.assert_allclose(meta["var"][p], ex2 - meta["mean"][p] ** 2, rtol=1e-9, atol=1e-9)
        assert meta["count"][p] == blk.shape[0]
    meta2 = pages.page_metadata(keys + 5.0, 32)
    np.testing.assert_allclose(meta2["var"], meta["var"], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(meta2["mean"], meta["mean"] + 5.0, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("ps,d", [(16, 64), (64, 128)])
def test_replica_meta_against_f64(ps, d):
    rng = np.random.default_rng(14)
    L = 5 * ps + 3
    keys = _keys(rng, L, d, ps)
    f = pages.page_metadata(keys, ps)
    r = replica.page_meta(keys, ps)
    # extremes are exact
    assert np.array_equal(r["kmin"].astype(np.float64), f["kmin"])
    assert np.array_equal(r["kmax"].astype(np.float64), f["kmax"])
    assert np.array_equal(r["count"], f["count"])
    np.testing.assert_allclose(r["mean"], f["mean"], rtol=0, atol=2e-6)
    var32 = r["m2"].astype(np.float64) / r["count"][:, None]
    np.testing.assert_allclose(var32, f["var"], rtol=1e-4, atol=1e-7)


def test_replica_incremental_equals_whole_page():
    """Welford state is (mean, m2, kmin, kmax): resuming a partial page from its
    stored fp32 state gives the same bits as processing it in one go."""
    rng = np.random.default_rng(15)
    ps, d = 16, 8
    keys = _keys(rng, 3 * ps, d, ps)
    whole = replica.page_meta(keys, ps)
    # emulate resuming: process the first 5 tokens of page 1, then the rest
    part = replica.page_meta(keys[ps:ps + 5], ps)
    mu, s = part["mean"][0].copy(), part["m2"][0].copy()
    lo, hi = part["kmin"][0].copy(), part["kmax"][0].copy()
    for t in range(5, ps):
        x = keys[ps + t].astype(np.float32)
        n = np.float32(t + 1)
        d1 = (x - mu).astype(np.float32)
        mu = (mu + (d1 / n).astype(np.float32)).astype(np.float32)
        d2 = (x - mu).astype(np.float32)
        s = (s.astype(np.float64) + d1.astype(np.float64) * d2.astype(np.float64)).astype(np.float32)
        lo = np.where(x < lo, x, lo)
        hi = np.where(x > hi, x, hi)
    assert np.array_equal(mu, whole["mean"][1])
    assert np.array_equal(lo, whole["kmin"][1]) and np.array_equal(hi, whole["kmax"][1])
    # the fused m2 step, done in float64 then rounded once, is fmaf exactly
    # (the product of two fp32 numbers is exact in float64, and a single
    # rounding of an exact sum to fp32 is the fmaf result unless the float64
    # sum itself rounded; allow that rare double-rounding ulp)
    np.testing.assert_array_max_ulp(s, whole["m2"][1], maxulp=1)


@pytest.mark.parametrize("ps,d", [(16, 64), (64, 128)])
def test_replica_gauss_against_f64(ps, d):
    rng = np.random.default_rng(16)
    L = 6 * ps + 1          # last page holds a single token
    keys = _keys(rng, L, d, ps)
    q = rng.standard_normal((4, d)).astype(np.float32)
    scale = float(np.float32(1.0 / np.sqrt(d)))
    f = pages.page_metadata(keys, ps)
    m64, v64 = pages.gauss_scores(q, f["mean"], f["var"], scale)
    r = replica.page_meta(keys, ps)
    m, v, est = replica.gauss(q, r["mean"], r["m2"], r["count"], scale, ps)
    np.testing.assert_allclose(m, m64, rtol=0, atol=2e-5)
    np.testing.assert_allclose(v, v64, rtol=2e-4, atol=1e-7)
    from oracle import gauss
    e64 = gauss.est_max(m64, v64, f["count"][None, :], ps)
    np.testing.assert_allclose(est, e64, rtol=0, atol=5e-5)
    # pages with one token have zero spread: the estimate is the mean score
    one = np.nonzero(r["count"] == 1)[0]
    assert one.size == 0 or np.array_equal(est[:, one], m[:, one])


def test_gauss_scores_are_the_score_moments_when_keys_vary_in_one_coordinate():
    """With keys that differ in a single coordinate the diagonal model is
    exact: m and v must equal the mean and population variance of the true
    scores scale * q.k over the page (pins scale^2 and q^2 in v)."""
    rng = np.random.default_rng(17)
    d, n, scale = 16, 23, 0.37
    for j in (0, 5, 15):
        c = rng.standard_normal(d)
        keys = np.tile(c, (n, 1))
        keys[:, j] += 2.0 * rng.standard_normal(n)
        q = rng.standard_normal((3, d))
        meta = pages.page_metadata(keys, n)
        m, v = pages.gauss_scores(q, meta["mean"], meta["var"], scale)
        s = scale * (keys @ q.T)                       # [n, heads]
        np.testing.assert_allclose(m[:, 0], s.mean(axis=0), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(v[:, 0], s.var(axis=0), rtol=1e-10, atol=1e-12)


def test_estimated_page_maximum_scales_with_the_spread():
    """est_max - m is proportional to the standard deviation sqrt(v) (scaling
    the scores by c scales it by c), zero for one token, and positive and
    increasing in the page's token count from two tokens on."""
    m = np.array([0.4, -1.0, 2.0])
    v = np.array([0.09, 0.25, 1.0])
    for n in (2, 3, 17, 64):
        nn = np.full(3, n)
        e1 = gauss.est_max(m, v, nn, 64) - m
        e4 = gauss.est_max(3.0 * m, 9.0 * v, nn, 64) - 3.0 * m
        np.testing.assert_allclose(e4, 3.0 * e1, rtol=1e-12)
        assert np.all(e1 > 0)
    grow = [float(gauss.est_max(m[:1], v[:1], np.array([n]), 64)[0]) for n in range(1, 65)]
    assert grow[0] == m[0] and all(a < b for a, b in zip(grow, grow[1:]))
