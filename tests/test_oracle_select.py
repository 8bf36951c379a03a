"""Pins of the selection oracle (c5, c6).

Top-k is checked against the properties that characterise it uniquely: the
set has min(k, P) members, every kept key is >= every dropped key, and among
keys equal to the smallest kept key the kept indices are the lowest.  The
Gaussian keep rule is checked on its degenerate cases.
"""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import entmax, select


def _check_topk(keys, k, sel):
    keys = np.asarray(keys, dtype=np.float32)
    P = keys.size
    assert len(sel) == min(k, P)
    assert list(sel) == sorted(set(int(i) for i in sel))
    kept = np.zeros(P, dtype=bool)
    kept[sel] = True
    if kept.any() and (~kept).any():
        kmin = keys[kept].min()
        assert keys[~kept].max() <= kmin
        ties = np.nonzero(keys == kmin)[0]
        kt = [i for i in ties if kept[i]]
        dt = [i for i in ties if not kept[i]]
        if kt and dt:
            assert max(kt) < min(dt)


@settings(max_examples=200, deadline=None)
@given(st.lists(st.sampled_from([-2.0, -0.0, 0.0, 0.5, 1.0, 1.0, 3.5, 7.25]), min_size=1, max_size=60),
       st.integers(min_value=0, max_value=70))
def test_topk_properties_with_ties(keys, k):
    _check_topk(keys, k, select.topk(keys, k))


def test_topk_random_and_planted():
    rng = np.random.default_rng(30)
    keys = rng.standard_normal(2048).astype(np.float32)
    keys[1234] = 100.0
    sel = select.topk(keys, 64)
    _check_topk(keys, 64, sel)
    assert 1234 in sel
    assert np.array_equal(select.topk(keys, 5000), np.arange(2048))


def test_signed_zero_ties_go_to_lower_index():
    keys = np.array([-0.0, 0.0, -0.0, -1.0], dtype=np.float32)
    assert list(select.topk(keys, 2)) == [0, 1]


@pytest.mark.parametrize("P,frac,k", [(16384, 1 / 64, 256), (100, 1 / 16, 7), (2048, 1 / 32, 64),
                                      (3, 1 / 16, 1), (0, 1 / 16, 0)])
def test_budget_fraction(P, frac, k):
    assert select.budget_pages(P, -1, frac) == k
    assert select.budget_pages(P, 5, frac) == min(5, P)


def test_gauss_keep_degenerate_cases():
    rng = np.random.default_rng(31)
    est = rng.standard_normal((4, 300)).astype(np.float32)
    tau = np.float32(0.5) * est.max(axis=1)
    assert np.array_equal(select.gauss_keep(est, tau, 1.5, 1e6), np.arange(300))
    # one token per page, zero spread: est is the exact score, and with
    # Delta = 0 the kept pages are exactly those holding a support token
    s = rng.standard_normal(300)
    est1 = s.astype(np.float32)[None, :]
    x = 0.5 * est1[0].astype(np.float64)
    p, t = entmax.probs(x, 1.5)
    kept = select.gauss_keep(est1, np.array([np.float32(t)]), 1.5, 0.0)
    support = np.nonzero(p > 0)[0]
    assert set(support) <= set(kept)
    assert len(kept) - len(support) <= 1     # at most a token sitting on tau


def test_gauss_keep_bands():
    est = np.array([[1.0, 2.0, 3.0]])
    keep, drop = select.gauss_keep_bands(est, np.array([1.0]), 1.5, 0.0, 0.1)
    # margins 0.5*est - 1 = -0.5, 0, 0.5
    assert list(keep) == [2] and list(drop) == [0]


def test_gauss_keep_threshold_is_inclusive_and_a_union_over_the_group():
    """A page is kept when (alpha-1) est reaches tau_hat - Delta (equality
    included, decided in fp32), and for a kv head when any query head of its
    group keeps it."""
    f = np.float32
    at = f(0.75)
    est = np.array([[at, np.nextafter(at, f(-1)), np.nextafter(at, f(2))]], dtype=np.float32)
    assert list(select.gauss_keep(est, np.array([f(1.0)]), 2.0, 0.25)) == [0, 2]
    est2 = np.array([[1.0, -3.0, -3.0, -3.0],
                     [-3.0, -3.0, 1.0, -3.0]], dtype=np.float32)
    tau = np.array([f(0.2), f(0.2)])
    assert list(select.gauss_keep(est2, tau, 1.5, 0.0)) == [0, 2]
    assert list(select.gauss_keep(est2[:1], tau[:1], 1.5, 0.0)) == [0]
