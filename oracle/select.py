"""Candidate page selection (test infrastructure only).

EntmaxKV pages, section 2.B (candidate selection policies):

1. top-k page selection: a fixed budget of the k pages with the highest
   bounding-box upper bounds;
2. Gaussian-aware entmax selection: keep the pages whose estimated maximum
   score clears tau_hat minus a safety margin Delta.

Readings (the pages leave these open):

* grouped-query attention: one page list serves a kv-head and its group of
  query heads.  Top-k ranks pages by the group's largest bound
  UBg_p = max_h UB_{h,p}; the Gaussian rule keeps the union over the group;
* ties in top-k go to the lower page index; -0 counts as +0;
* a budget given as a fraction f of the P pages means k = ceil(f * P)
  (f read as float32, product taken in float64), clipped to P;
* the emitted list is sorted by page index.

The keys handed to these functions are the fp32 values from ``replica``; the
decisions are taken in fp32 exactly as written here.
"""

import math

import numpy as np


def budget_pages(P, budget, frac):
    """Number of pages to keep for a sequence with P pages."""
    if budget >= 0:
        k = int(budget)
    else:
        k = int(math.ceil(float(np.float32(frac)) * float(P)))
    return max(0, min(k, int(P)))


def topk(keys, k):
    """Indices of the k largest keys (ties -> lower index), sorted ascending."""
    keys = np.asarray(keys, dtype=np.float32)
    P = keys.size
    k = min(int(k), P)
    order = sorted(range(P), key=lambda i: (-float(keys[i]), i))
    return np.array(sorted(order[:k]), dtype=np.int64)


def gauss_keep(est, tau_hat, alpha, delta):
    """Pages kept by the Gaussian rule, decided in fp32.

    est: [G, P] fp32 estimated page maxima (score space); tau_hat: [G] fp32.
    Page p is kept iff for some head h: fp32((alpha-1) * est[h, p]) >=
    fp32(tau_hat[h] - delta).
    """
    est = np.asarray(est, dtype=np.float32)
    tau_hat = np.asarray(tau_hat, dtype=np.float32)
    am1 = np.float32(alpha - 1.0)
    lhs = (am1 * est).astype(np.float32)
    rhs = (tau_hat - np.float32(delta)).astype(np.float32)
    keep = np.any(lhs >= rhs[:, None], axis=0)
    return np.nonzero(keep)[0].astype(np.int64)


def gauss_keep_bands(est, tau_hat64, alpha, delta, band):
    """(must_keep, must_drop) page sets for a float64 threshold.

    A page whose margin (alpha-1) est - (tau_hat - delta) is above +band for
    some head must be kept; one whose margin is below -band for every head
    must be dropped; anything in between may go either way.
    """
    est = np.asarray(est, dtype=np.float64)
    tau_hat64 = np.asarray(tau_hat64, dtype=np.float64)
    margin = (alpha - 1.0) * est - (tau_hat64[:, None] - delta)
    must_keep = np.nonzero(np.any(margin > band, axis=0))[0]
    must_drop = np.nonzero(np.all(margin < -band, axis=0))[0]
    return must_keep, must_drop
