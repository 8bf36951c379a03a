"""Entmax attention over kept tokens and the full-cache baselines (float64).

Test infrastructure only.

EntmaxKV pages, section 2.C (sparse entmax attention): once candidate pages are
chosen only their keys and values are loaded and alpha-entmax is computed over
that reduced set; if the set contains the full support the output is exact.
Section 3: the output error is bounded by 2 B delta, B a bound on the value
norms and delta the probability mass of the dropped tokens; for alpha-entmax
delta = 0 whenever the kept set contains the support S.  Section 4 compares
against full-cache softmax (FlashDecoding) and full-cache entmax decoding.

Definitions used:

* scores s_i = scale * q . k_i, entmax inputs x_i = (alpha - 1) s_i;
* p = alpha-entmax(x) over the kept tokens only (the threshold is re-solved on
  the kept set);
* o = sum_i p_i v_i, accumulated in ascending token index over the tokens with
  p_i > 0 (adding an exact zero changes nothing, so this is the full sum);
* softmax baseline: o = sum_i softmax(s)_i v_i.
"""

import numpy as np

from . import entmax


def _acc(p, V):
    """sum_i p_i V[i] over p_i > 0, ascending i, float64."""
    out = np.zeros(V.shape[1])
    for i in np.nonzero(p > 0)[0]:
        out = out + p[i] * V[i]
    return out


def _scores(q, K):
    """q . k_i per token and head, each a row sum of elementwise products.

    A per-row reduction does not depend on how many other rows there are
    (unlike a blocked matrix product), so a token gets the same score whether
    it is scored with the whole cache or with a subset.
    """
    return np.stack([(K * q[h][None, :]).sum(axis=1) for h in range(q.shape[0])], axis=1)


def entmax_attention(q, K, V, alpha, scale, method="sort"):
    """Exact alpha-entmax attention of G query heads over n tokens.

    q: [G, d]; K, V: [n, d] (bf16 values widened exactly, or fp32).
    Returns (o [G, d], tau [G], p [G, n]).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    G = q.shape[0]
    x = (alpha - 1.0) * scale * _scores(q, K)  # [n, G]
    o = np.zeros((G, V.shape[1]))
    tau = np.zeros(G)
    P = np.zeros((G, K.shape[0]))
    for h in range(G):
        p, t = entmax.probs(x[:, h], alpha, method)
        P[h] = p
        tau[h] = t
        o[h] = _acc(p, V)
    return o, tau, P


def softmax_attention(q, K, V, scale):
    """Full softmax attention of G heads over n tokens, float64."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    s = scale * _scores(q, K)
    o = np.zeros((q.shape[0], V.shape[1]))
    for h in range(q.shape[0]):
        o[h] = entmax.softmax(s[:, h]) @ V
    return o


def token_indices(pages, seq_len, ps):
    """Logical token indices of the given pages (ascending), clipped to seq_len."""
    idx = []
    for p in sorted(int(x) for x in pages):
        idx.extend(range(p * ps, min(seq_len, (p + 1) * ps)))
    return np.asarray(idx, dtype=np.int64)


def dropped_mass(p_full, kept_tokens):
    """delta = total full-cache probability of tokens outside the kept set."""
    keep = np.zeros(p_full.shape[-1], dtype=bool)
    keep[kept_tokens] = True
    return p_full[..., ~keep].sum(axis=-1)


def support_recall(p_full, kept_tokens):
    """|S intersect I_keep| / |S| per head, S = {i : p_i > 0}."""
    keep = np.zeros(p_full.shape[-1], dtype=bool)
    keep[kept_tokens] = True
    S = p_full > 0
    return (S & keep[None, :]).sum(axis=-1) / np.maximum(S.sum(axis=-1), 1)
