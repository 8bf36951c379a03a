"""Per-page metadata and page scores in float64 (test infrastructure only).

EntmaxKV pages, section 2.A (query-aware page scoring): the KV cache is split
into pages; before any key or value is loaded every page is scored from small
metadata kept per page:

* a bounding box, the coordinatewise minimum and maximum key (k_min, k_max),
  which gives a deterministic upper bound on q.k for every key in the page;
* the first and second moments (mean and variance) of the page's keys, which
  model the scores inside the page as a Gaussian.

Readings (the pages give no formula):

* bound: UB_p(q) = scale * sum_d max(q_d k_min[d], q_d k_max[d]), the largest
  value of scale * q.k over the box, hence >= every true score in the page;
* variance: per coordinate (diagonal), population variance (divide by n);
* page score model: m_p = scale * q.mu_p, v_p = scale^2 * sum_d q_d^2 var_p[d];
* a page holds only the tokens written so far (the last page may be partial).
"""

import numpy as np


def n_pages(seq_len, ps):
    return (int(seq_len) + ps - 1) // ps


def page_metadata(keys, ps):
    """Metadata of every logical page of one (sequence, kv-head).

    keys: [L, d] key vectors in logical token order.
    Returns dict with kmin, kmax, mean, var ([P, d] float64) and count ([P]).
    """
    keys = np.asarray(keys, dtype=np.float64)
    L, d = keys.shape
    P = n_pages(L, ps)
    out = {k: np.zeros((P, d)) for k in ("kmin", "kmax", "mean", "var")}
    out["count"] = np.zeros(P, dtype=np.int64)
    for p in range(P):
        blk = keys[p * ps:min(L, (p + 1) * ps)]
        out["kmin"][p] = blk.min(axis=0)
        out["kmax"][p] = blk.max(axis=0)
        out["mean"][p] = blk.mean(axis=0)
        out["var"][p] = ((blk - blk.mean(axis=0)) ** 2).mean(axis=0)
        out["count"][p] = blk.shape[0]
    return out


def bbox_bound(q, kmin, kmax, scale):
    """UB[h, p] = scale * sum_d max(q[h,d] kmin[p,d], q[h,d] kmax[p,d])."""
    q = np.asarray(q, dtype=np.float64)
    kmin = np.asarray(kmin, dtype=np.float64)
    kmax = np.asarray(kmax, dtype=np.float64)
    lo = q[:, None, :] * kmin[None, :, :]
    hi = q[:, None, :] * kmax[None, :, :]
    return scale * np.maximum(lo, hi).sum(axis=2)


def gauss_scores(q, mean, var, scale):
    """(m, v)[h, p]: mean and variance of scale * q.k for k ~ N(mu_p, diag var_p)."""
    q = np.asarray(q, dtype=np.float64)
    m = scale * (q @ np.asarray(mean, dtype=np.float64).T)
    v = scale * scale * ((q * q) @ np.asarray(var, dtype=np.float64).T)
    return m, v


def true_page_max(q, keys, ps, scale):
    """max over the tokens of each page of scale * q.k, [h, P] (for checks)."""
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    s = scale * (keys @ q.T)            # [L, h]
    L = keys.shape[0]
    P = n_pages(L, ps)
    out = np.empty((q.shape[0], P))
    for p in range(P):
        out[:, p] = s[p * ps:min(L, (p + 1) * ps)].max(axis=0)
    return out
