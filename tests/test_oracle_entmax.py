"""Pins of the float64 alpha-entmax oracle (c1) to things other than itself.

* hand-derived worked examples (tests/golden/worked_examples.json);
* the variational definition of alpha-entmax (maximiser of
  p.s + (1/(alpha(alpha-1))) sum_j (p_j - p_j^alpha) on the simplex, with the
  raw score s = x / (alpha - 1)), solved
  by a general-purpose constrained optimiser;
* brute force over all supports for n <= 8 with a scalar root finder;
* invariants (sum p = 1, p >= 0, shift equivariance) and the alpha -> 1 limit
  (softmax).
"""
import itertools
import json
import os

import numpy as np
import pytest
from scipy.optimize import brentq, minimize

from oracle import entmax

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


@pytest.mark.parametrize("ex", GOLD["entmax"], ids=lambda e: e["name"])
def test_worked_examples(ex):
    x = np.array(ex["x"])
    for method in ("sort", "bisect"):
        p, tau = entmax.probs(x, ex["alpha"], method)
        assert abs(tau - ex["tau"]) < 1e-12
        np.testing.assert_allclose(p, ex["p"], atol=1e-12)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_sort_and_bisect_agree(alpha):
    rng = np.random.default_rng(1)
    for n in (1, 2, 3, 17, 256, 4096):
        for scale in (0.1, 1.0, 10.0):
            x = scale * rng.standard_normal(n)
            t1 = entmax.tau_sort(x, alpha)
            t2 = entmax.tau_bisect(x, alpha)
            assert abs(t1 - t2) < 1e-12 * max(1.0, abs(t1))


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 3.0])
def test_simplex_and_shift(alpha):
    rng = np.random.default_rng(2)
    x = rng.standard_normal(300)
    p, tau = entmax.probs(x, alpha)
    assert (p >= 0).all()
    assert abs(p.sum() - 1.0) < 1e-12
    p2, tau2 = entmax.probs(x + 3.25, alpha)
    np.testing.assert_allclose(p2, p, atol=1e-12)
    assert abs(tau2 - tau - 3.25) < 1e-11
    # exact zeros below the threshold, positive above
    assert np.all((p > 0) == (x > tau))


def _variational(x, alpha):
    """argmax_p p.s + (1/(alpha(alpha-1))) sum(p - p^alpha) on the simplex,
    s = x / (alpha - 1) the raw score (the solution is [x - tau]_+^(1/(alpha-1)))."""
    s = x / (alpha - 1.0)
    n = x.size

    def neg(p):
        p = np.clip(p, 0.0, None)
        return -(p @ s + (p - p ** alpha).sum() / (alpha * (alpha - 1.0)))

    best = None
    for start in (np.full(n, 1.0 / n), np.eye(n)[int(np.argmax(s))] * 0.9 + 0.1 / n):
        res = minimize(neg, start, method="SLSQP", bounds=[(0.0, 1.0)] * n,
                       constraints=[{"type": "eq", "fun": lambda p: p.sum() - 1.0}],
                       options={"ftol": 1e-15, "maxiter": 500})
        if best is None or res.fun < best.fun:
            best = res
    return np.clip(best.x, 0.0, None)


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25, 3.0])
def test_variational_definition(alpha):
    rng = np.random.default_rng(3)
    for _ in range(6):
        x = rng.standard_normal(5)
        p, _ = entmax.probs(x, alpha)
        q = _variational(x, alpha)
        np.testing.assert_allclose(p, q, atol=2e-5)


def _brute_force(x, alpha):
    """Enumerate supports S; keep the one whose root tau of sum_S (x-tau)^r = 1
    satisfies min_S x > tau >= max_{not S} x."""
    r = 1.0 / (alpha - 1.0)
    n = x.size
    found = []
    for size in range(1, n + 1):
        for S in itertools.combinations(range(n), size):
            S = list(S)
            xs = x[S]
            f = lambda t: np.sum((xs - t) ** r) - 1.0   # noqa: E731
            hi = xs.min()
            lo = xs.max() - 1.0 - 1e-9
            if f(hi) > 0 or f(lo) < 0:
                continue
            tau = brentq(f, lo, hi, xtol=1e-15, rtol=1e-15)
            rest = np.delete(x, S)
            if (xs > tau).all() and (rest.size == 0 or rest.max() <= tau + 1e-14):
                found.append(tau)
    assert found, "no consistent support"
    tau = found[0]
    for t in found[1:]:
        assert abs(t - tau) < 1e-9        # uniqueness
    return tau


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.7, 1.25, 3.0])
def test_brute_force_supports(alpha):
    rng = np.random.default_rng(4)
    for n in range(1, 9):
        x = 0.7 * rng.standard_normal(n)
        tau = _brute_force(x, alpha)
        p, t = entmax.probs(x, alpha)
        assert abs(t - tau) < 1e-9
        np.testing.assert_allclose(p, np.maximum(x - tau, 0) ** (1 / (alpha - 1)), atol=1e-9)


def test_softmax_limit():
    rng = np.random.default_rng(5)
    s = rng.standard_normal(40)
    sm = entmax.softmax(s)
    errs = []
    for a in (1.1, 1.01, 1.001):
        p, _ = entmax.probs((a - 1.0) * s, a)
        errs.append(np.abs(p - sm).max())
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 5e-3


def test_sparsemax_two_entries_closed_form():
    # textbook: sparsemax([a, b])_1 = clip((a - b + 1) / 2, 0, 1)
    for a, b in [(0.0, 0.0), (0.3, -0.1), (2.0, 0.0), (-0.4, 0.4), (0.9, 0.1)]:
        p, _ = entmax.probs(np.array([a, b]), 2.0)
        assert abs(p[0] - min(1.0, max(0.0, (a - b + 1.0) / 2.0))) < 1e-14
