"""Gaussian-aware threshold estimate tau_hat in float64 (test infrastructure only).

EntmaxKV pages, section 2.B, policy 2 (Gaussian-aware entmax selection): the
global alpha-entmax threshold is estimated from page-level Gaussian
statistics by solving an approximate normalisation equation for tau_hat; a
page is kept when its estimated maximum score clears tau_hat minus a safety
margin Delta.  The abstract adds that the estimate comes from lightweight page
statistics and adapts the budget to the score distribution.

The pages print neither the equation nor the page-maximum estimator.  Reading
taken here (the plainest one consistent with the entmax definition):

* every token of page p has score s ~ N(m_p, v_p), so x = (alpha-1) s is
  N(m'_p, sigma'_p^2) with m' = (alpha-1) m and sigma' = (alpha-1) sqrt(v);
* tau_hat solves the expected entmax normalisation over all tokens,

      F(tau) = sum_p n_p * E[(X_p - tau)_+^(1/(alpha-1))] = 1,

  n_p the number of tokens in page p; with u = m' - tau and z = u / sigma':
      alpha = 2:   E[(X - tau)_+]   = u Phi(z) + sigma' phi(z)
      alpha = 1.5: E[(X - tau)_+^2] = (u^2 + sigma'^2) Phi(z) + u sigma' phi(z)
      other alpha: numerical integration (adaptive quadrature)
      sigma' = 0:  max(u, 0)^(1/(alpha-1));
* the estimated page maximum is the Gaussian expected-maximum approximation
  est_max_p = m_p + sqrt(v_p) * z_{n_p}, z_n = sqrt(2 ln n) (z_1 = 0), i.e. a
  statistic built from the page's mean and spread (Hindi summary, the
  "weather forecast" analogy of the Gaussian selector);
* Delta is measured in the same x = (alpha-1) s space as tau.

F is continuous and strictly decreasing wherever it is positive, so tau_hat is
found by bisection on a bracket grown by doubling steps.
"""

import math

import numpy as np
from scipy.integrate import quad
from scipy.special import ndtr


def _phi(z):
    return np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def _g_quad(u, s, r):
    """E[(Y)_+^r] for Y ~ N(u, s^2), s > 0, by adaptive quadrature.

    With z = u / s the expectation is s^r * int_0^inf y^r phi(y - z) dy.  The
    log of the integrand, r ln y - (y - z)^2 / 2, is concave (second derivative
    -(1 + r / y^2) <= -1) with its peak at y* = (z + sqrt(z^2 + 4 r)) / 2, so the
    integrand is below exp(-72) of its peak outside |y - y*| <= 12; [0, ...] is
    integrated with the quadrature's algebraic endpoint weight for y^r."""
    z = u / s
    ys = 0.5 * (z + math.sqrt(z * z + 4.0 * r))
    lo, hi = max(0.0, ys - 12.0), ys + 12.0
    if lo == 0.0:
        val, _ = quad(lambda y: _phi(y - z), 0.0, hi, weight="alg", wvar=(r, 0.0),
                      epsabs=0.0, epsrel=1e-12, limit=400)
    else:
        val, _ = quad(lambda y: y ** r * _phi(y - z), lo, hi, points=[ys], epsabs=0.0, epsrel=1e-12,
                      limit=400)
    return s ** r * val


def g(mp, sp, tau, alpha, method="closed"):
    """E[(X - tau)_+^(1/(alpha-1))] for X ~ N(mp, sp^2), elementwise, float64.

    alpha = 1.5 and 2 have closed forms; any other alpha (or method="quad")
    integrates numerically."""
    mp = np.asarray(mp, dtype=np.float64)
    sp = np.asarray(sp, dtype=np.float64)
    u = mp - tau
    r = 1.0 / (alpha - 1.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(sp > 0, u / np.where(sp > 0, sp, 1.0), 0.0)
    if method == "closed" and alpha == 2.0:
        gauss = u * ndtr(z) + sp * _phi(z)
    elif method == "closed" and alpha == 1.5:
        gauss = (u * u + sp * sp) * ndtr(z) + u * sp * _phi(z)
    else:
        uu, ss = np.broadcast_arrays(u, sp)
        gauss = np.array([_g_quad(a, b, r) if b > 0 else 0.0 for a, b in zip(uu.ravel(), ss.ravel())])
        gauss = gauss.reshape(uu.shape)
    point = np.maximum(u, 0.0) ** r
    return np.where(sp > 0, gauss, point)


def F(tau, m, v, n, alpha):
    """Expected entmax mass sum_p n_p E[(X_p - tau)_+^r] for page scores (m, v)."""
    am1 = alpha - 1.0
    mp = am1 * np.asarray(m, dtype=np.float64)
    sp = am1 * np.sqrt(np.maximum(np.asarray(v, dtype=np.float64), 0.0))
    return float(np.sum(np.asarray(n, dtype=np.float64) * g(mp, sp, tau, alpha)))


def tau_hat(m, v, n, alpha, iters=100):
    """Root of F(tau) = 1 by bisection (float64)."""
    am1 = alpha - 1.0
    m = np.asarray(m, dtype=np.float64)
    v = np.maximum(np.asarray(v, dtype=np.float64), 0.0)
    if m.size == 0:
        raise ValueError("tau_hat of an empty page set")
    mp = am1 * m
    sp = am1 * np.sqrt(v)
    hi = float(np.max(mp + 8.0 * sp))
    step = 1.0
    while F(hi, m, v, n, alpha) > 1.0:
        hi += step
        step *= 2.0
    lo = hi - 1.0
    step = 1.0
    while F(lo, m, v, n, alpha) < 1.0:
        lo -= step
        step *= 2.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if F(mid, m, v, n, alpha) >= 1.0:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def z_table(ps):
    """z_n = sqrt(2 ln n) for n >= 2, z_0 = z_1 = 0; length ps + 1, float64."""
    z = np.zeros(ps + 1)
    for n in range(2, ps + 1):
        z[n] = math.sqrt(2.0 * math.log(n))
    return z


def est_max(m, v, n, ps):
    """Estimated page maximum score m + sqrt(v) z_n (float64)."""
    z = z_table(ps)
    return np.asarray(m, dtype=np.float64) + np.sqrt(np.maximum(v, 0.0)) * z[np.asarray(n)]
