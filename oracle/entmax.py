"""alpha-entmax in float64 (test infrastructure only).

EntmaxKV pages, section 2 (methodology): for alpha > 1, alpha-entmax yields a
probability distribution with exact zeros, so sparse decoding that keeps the
support is exact.  The pages do not write the map out; the definition used
here is the standard one

    p_i = [x_i - tau]_+ ^ (1 / (alpha - 1)),   tau unique with sum_i p_i = 1,

where x_i = (alpha - 1) * s_i and s_i is the attention score.

Two independent ways to find tau are given:

* ``tau_bisect``: bisection on the monotone map tau -> sum_i [x_i - tau]_+^r
  over the bracket [max x - 1, max x - n^(1 - alpha)] (the mass is >= 1 at the
  left end because the top term alone is 1, and <= 1 at the right end because
  every term is <= 1/n).
* ``tau_sort`` (alpha in {1.5, 2} only): sort x in decreasing order and, for
  each prefix size k, solve the normalisation equation restricted to the top
  k entries in closed form; the support size is the largest k whose solution
  lies below the k-th largest entry.  For alpha = 2 this is sparsemax
  (tau_k = (sum_{j<=k} x_j - 1) / k); for alpha = 1.5 the restricted equation
  sum_{j<=k} (x_j - tau)^2 = 1 is a quadratic whose smaller root is
  tau_k = M_k - sqrt(M_k^2 - S_k + 1/k), M_k and S_k the mean and mean square
  of the top k entries.
"""

import numpy as np


def _r(alpha):
    if not alpha > 1.0:
        raise ValueError("alpha-entmax needs alpha > 1")
    return 1.0 / (alpha - 1.0)


def mass(x, tau, alpha):
    """sum_i [x_i - tau]_+^(1/(alpha-1)) in float64."""
    x = np.asarray(x, dtype=np.float64)
    return float(np.sum(np.maximum(x - tau, 0.0) ** _r(alpha)))


def tau_bisect(x, alpha, iters=200):
    """Threshold by bisection (any alpha > 1)."""
    x = np.asarray(x, dtype=np.float64).ravel()
    x = x[np.isfinite(x)]
    n = x.size
    if n == 0:
        raise ValueError("entmax of an empty vector")
    r = _r(alpha)
    top = float(x.max())
    lo = top - 1.0
    hi = top - float(n) ** (1.0 - alpha)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if np.sum(np.maximum(x - mid, 0.0) ** r) >= 1.0:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def tau_sort(x, alpha):
    """Exact threshold by the sorted-prefix closed form (alpha in {1.5, 2})."""
    x = np.asarray(x, dtype=np.float64).ravel()
    x = x[np.isfinite(x)]
    n = x.size
    if n == 0:
        raise ValueError("entmax of an empty vector")
    z = np.sort(x)[::-1]
    k = np.arange(1, n + 1, dtype=np.float64)
    csum = np.cumsum(z)
    if alpha == 2.0:
        tau_k = (csum - 1.0) / k
        ok = tau_k < z
    elif alpha == 1.5:
        mean = csum / k
        msq = np.cumsum(z * z) / k
        disc = mean * mean - msq + 1.0 / k
        valid = disc >= 0.0
        tau_k = np.where(valid, mean - np.sqrt(np.where(valid, disc, 0.0)), np.inf)
        ok = valid & (tau_k < z)
    else:
        raise ValueError("closed form only for alpha in {1.5, 2}")
    # the largest prefix whose threshold sits below its own last entry
    ks = np.nonzero(ok)[0]
    return float(tau_k[ks[-1]])


def probs(x, alpha, method="sort"):
    """(p, tau) of alpha-entmax; non-finite x (masked slots) get p = 0."""
    x = np.asarray(x, dtype=np.float64)
    if method == "sort" and alpha in (1.5, 2.0):
        tau = tau_sort(x, alpha)
    else:
        tau = tau_bisect(x, alpha)
    with np.errstate(invalid="ignore"):
        p = np.where(np.isfinite(x), np.maximum(x - tau, 0.0), 0.0) ** _r(alpha)
    return p, tau


def softmax(s):
    """Plain softmax in float64."""
    s = np.asarray(s, dtype=np.float64)
    e = np.exp(s - s.max())
    return e / e.sum()
