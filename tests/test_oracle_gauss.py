"""Pins of the Gaussian tau_hat oracle (c4, c5).

* closed-form page expectations g against numerical integration (scipy quad)
  and against Monte-Carlo (10^6 draws, 4-sigma bound), and against the worked
  examples in tests/golden;
* with one token per page and zero spread, F is the exact entmax mass, so
  tau_hat must equal the exact entmax threshold of c1; with n equal tokens
  per page it is the threshold of the multiset repeating each page n times;
* F against a Monte-Carlo over the token scores in score space, which fixes
  the map (m, v) -> ((alpha-1) m, (alpha-1) sqrt(v)) of the entmax input;
* F is strictly decreasing and F(tau_hat) = 1;
* the z table against sqrt(2 ln n).
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.integrate import quad

from oracle import entmax, gauss

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


@pytest.mark.parametrize("ex", GOLD["gauss_g"], ids=lambda e: "a%g_m%g_s%g" % (e["alpha"], e["m"], e["s"]))
def test_g_worked_examples(ex):
    val = gauss.g(ex["m"], ex["s"], ex["tau"], ex["alpha"])
    assert abs(float(val) - ex["g"]) < 1e-14


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25, 3.0, 1.1, 1.05])
def test_g_against_quadrature(alpha):
    r = 1.0 / (alpha - 1.0)
    for m, s, tau in [(0.3, 0.25, 0.9), (1.8, 0.15, 1.9), (-1.0, 2.0, 0.5), (0.0, 1e-3, -0.01),
                      (2.0, 0.5, 0.0), (0.1, 0.3, 2.5)]:
        dens = lambda x: math.exp(-0.5 * ((x - m) / s) ** 2) / (s * math.sqrt(2 * math.pi))  # noqa: E731
        val, err = quad(lambda x: (x - tau) ** r * dens(x), tau, max(tau, m) + 40 * s,
                        epsabs=1e-15, epsrel=1e-12, limit=400)
        assert abs(float(gauss.g(m, s, tau, alpha)) - val) < 1e-10 + 1e-9 * abs(val)


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25, 1.8, 3.0, 1.1])
def test_g_against_monte_carlo(alpha):
    rng = np.random.default_rng(20)
    r = 1.0 / (alpha - 1.0)
    for m, s, tau in [(0.5, 0.4, 0.6), (0.0, 1.0, -0.3)]:
        x = m + s * rng.standard_normal(1_000_000)
        y = np.maximum(x - tau, 0.0) ** r
        se = y.std() / math.sqrt(y.size)
        assert abs(y.mean() - float(gauss.g(m, s, tau, alpha))) < 4 * se


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25, 3.0, 1.1])
def test_point_pages_reduce_to_exact_entmax(alpha):
    rng = np.random.default_rng(21)
    for n in (1, 5, 64, 1000):
        s = rng.standard_normal(n)
        tau = gauss.tau_hat(s, np.zeros(n), np.ones(n), alpha)
        exact = entmax.tau_bisect((alpha - 1.0) * s, alpha)
        assert abs(tau - exact) < 1e-10


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_quadrature_path_matches_closed_forms(alpha):
    """The numerical path used for alpha outside {1.5, 2}, forced at 1.5 and 2."""
    m = np.array([0.3, 1.8, -1.0, 0.0, 2.0, 0.1, 5.0, -3.0])
    s = np.array([0.25, 0.15, 2.0, 1e-3, 0.5, 0.3, 0.01, 0.2])
    for tau in (-0.5, 0.0, 0.9, 1.9, 2.5):
        a = gauss.g(m, s, tau, alpha, method="closed")
        b = gauss.g(m, s, tau, alpha, method="quad")
        np.testing.assert_allclose(b, a, rtol=1e-9, atol=1e-14)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_F_decreasing_and_root(alpha):
    rng = np.random.default_rng(22)
    P = 500
    m = rng.standard_normal(P)
    v = (0.5 * rng.random(P)) ** 2
    n = rng.integers(1, 65, P)
    t = gauss.tau_hat(m, v, n, alpha)
    assert abs(gauss.F(t, m, v, n, alpha) - 1.0) < 1e-9
    grid = np.linspace(t - 2, t + 2, 81)
    vals = [gauss.F(x, m, v, n, alpha) for x in grid]
    assert all(a > b for a, b in zip(vals, vals[1:]))


@pytest.mark.parametrize("alpha", [1.25, 3.0, 1.1, 1.05])
def test_F_decreasing_and_root_any_alpha(alpha):
    rng = np.random.default_rng(23)
    P = 24
    m = rng.standard_normal(P)
    v = (0.5 * rng.random(P)) ** 2
    n = rng.integers(1, 65, P)
    t = gauss.tau_hat(m, v, n, alpha, iters=60)
    assert abs(gauss.F(t, m, v, n, alpha) - 1.0) < 1e-8
    vals = [gauss.F(x, m, v, n, alpha) for x in np.linspace(t - 1, t + 1, 9)]
    assert all(a > b for a, b in zip(vals, vals[1:]))


def test_z_table():
    for e in GOLD["z_table"]:
        assert abs(gauss.z_table(64)[e["n"]] - e["z"]) < 1e-15


def test_est_max_single_token_equals_mean():
    m = np.array([[0.3, -1.2]])
    v = np.array([[0.0, 0.0]])
    np.testing.assert_array_equal(gauss.est_max(m, v, np.array([[1, 1]]), 64), m)


@pytest.mark.parametrize("alpha", [1.5, 2.0, 3.0])
def test_pages_of_equal_tokens_reduce_to_exact_entmax_of_the_multiset(alpha):
    """A page whose n tokens share one score (zero spread) weighs that score n
    times: tau_hat equals the exact entmax threshold of the multiset in which
    every page's score is repeated n_p times (pins the n_p weighting)."""
    rng = np.random.default_rng(24)
    s = rng.standard_normal(40)
    n = rng.integers(1, 65, 40)
    tau = gauss.tau_hat(s, np.zeros(40), n, alpha)
    exact = entmax.tau_bisect((alpha - 1.0) * np.repeat(s, n), alpha)
    assert abs(tau - exact) < 1e-10
    # and it differs from the one-token-per-page threshold whenever n is not all ones
    assert abs(tau - entmax.tau_bisect((alpha - 1.0) * s, alpha)) > 1e-3


@pytest.mark.parametrize("alpha", [1.5, 2.0, 3.0])
def test_F_is_the_expected_mass_of_the_page_draws(alpha):
    """F(tau) = sum_p n_p E[((alpha-1) s - tau)_+^(1/(alpha-1))] with s ~ N(m_p, v_p)
    in score space: Monte-Carlo over the token scores themselves (pins the map
    from a page's score mean and variance to the entmax input's, (alpha-1) m and
    (alpha-1) sqrt(v))."""
    rng = np.random.default_rng(25)
    P = 6
    m = rng.uniform(-0.5, 2.0, P)
    v = rng.uniform(0.05, 0.8, P)
    n = rng.integers(1, 65, P)
    r = 1.0 / (alpha - 1.0)
    draws = 400_000
    for tau in (0.2, 0.6):
        est, var = 0.0, 0.0
        for p in range(P):
            x = (alpha - 1.0) * (m[p] + math.sqrt(v[p]) * rng.standard_normal(draws))
            y = n[p] * np.maximum(x - tau, 0.0) ** r
            est += y.mean()
            var += y.var() / draws
        assert abs(gauss.F(tau, m, v, n, alpha) - est) < 4.5 * math.sqrt(var)


def test_z_bounds_the_expected_maximum_of_n_normals():
    """z_n = sqrt(2 ln n) is the textbook upper bound on E[max of n independent
    standard normals] (from E[max] <= ln(n E[exp(t X)]) / t at t = z_n), and
    not far above it at page sizes: the estimate adds a spread-proportional
    margin of the right size to the page mean."""
    rng = np.random.default_rng(26)
    z = gauss.z_table(64)
    for n in (4, 16, 64):
        mx = rng.standard_normal((100_000, n)).max(axis=1)
        mean, se = mx.mean(), mx.std() / math.sqrt(mx.size)
        assert mean - 4 * se <= z[n] <= 1.7 * (mean + 4 * se)


@pytest.mark.parametrize("alpha", [1.1, 1.05])
def test_quadrature_follows_the_peak_of_large_powers(alpha):
    """For r = 1/(alpha-1) large, the integrand y^r phi(y - z) peaks at
    y* = (z + sqrt(z^2 + 4r)) / 2, well above z: the expectation must keep the
    mass there.  Against the same integral over the whole half line, with the
    peak given to the integrator, and against the closed form of the raw
    moments for z = 0 (E[Y_+^r] = 2^(r/2 - 1) Gamma((r + 1)/2) / sqrt(pi))."""
    r = 1.0 / (alpha - 1.0)
    for z in (-3.0, 0.0, 2.0):
        ys = 0.5 * (z + math.sqrt(z * z + 4.0 * r))
        f = lambda y: y ** r * math.exp(-0.5 * (y - z) ** 2) / math.sqrt(2 * math.pi)  # noqa: E731
        val = quad(f, 0.0, ys, epsabs=0.0, epsrel=1e-13, limit=400)[0] + \
            quad(f, ys, ys + 60.0, epsabs=0.0, epsrel=1e-13, limit=400)[0]
        got = float(gauss.g(z, 1.0, 0.0, alpha))
        assert abs(got - val) <= 1e-9 * val
    moment = 2 ** (r / 2 - 1) * math.gamma((r + 1) / 2) / math.sqrt(math.pi)
    assert abs(float(gauss.g(0.0, 1.0, 0.0, alpha)) - moment) <= 1e-9 * moment
