"""Pins of the attention oracle (c7, c8).

* support recovery is exact: if the kept tokens contain the entmax support,
  the sparse output equals the full-cache output (pages, section 3) -- bit for
  bit with the closed-form threshold (alpha 1.5, 2), to 1e-12 with bisection;
* the error bound ||o - o~|| <= 2 B delta when support tokens are dropped;
* o equals P @ V computed by a matrix product (a different summation order);
* softmax baseline: equal scores give the mean value vector; a dominating
  score gives that token's value;
* two tokens at alpha = 2 follow the textbook sparsemax closed form, and at
  alpha = 1.5 the quadratic solved by hand on x = (alpha - 1) scale q.k;
* softmax over a kept subset equals the full softmax weights restricted to
  the subset and renormalised, and obeys the same 2 B delta bound with a
  positive delta whenever a token is dropped (section 3);
* the support recovery and error bound also hold at alpha = 1.25 and 3.
"""
import numpy as np
import pytest

from oracle import attend


def _data(rng, n, d, G=4):
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    return q, K, V


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25, 3.0])
def test_support_recovery_is_bitwise_exact(alpha):
    rng = np.random.default_rng(40)
    q, K, V = _data(rng, 512, 32)
    scale = 1.0 / np.sqrt(32)
    o_full, tau_full, P = attend.entmax_attention(q, K, V, alpha, scale)
    support = np.nonzero(P.sum(axis=0) > 0)[0]
    assert 0 < support.size < 512
    extra = rng.choice(np.setdiff1d(np.arange(512), support), 40, replace=False)
    keep = np.sort(np.concatenate([support, extra]))
    o_sp, tau_sp, _ = attend.entmax_attention(q, K[keep], V[keep], alpha, scale)
    if alpha in (1.5, 2.0):     # closed form: the same prefix sums give the same tau, bit for bit
        assert np.array_equal(o_sp, o_full)
        assert np.array_equal(tau_sp, tau_full)
    else:                       # bisection: the bracket depends on n, so the last bits may differ
        np.testing.assert_allclose(o_sp, o_full, rtol=0, atol=1e-12)
        np.testing.assert_allclose(tau_sp, tau_full, rtol=0, atol=1e-12)
    assert np.all(attend.dropped_mass(P, keep) == 0)
    assert np.all(attend.support_recall(P, keep) == 1)


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25, 3.0])
def test_error_bound_when_support_is_dropped(alpha):
    rng = np.random.default_rng(41)
    q, K, V = _data(rng, 400, 16)
    scale = 0.25
    o_full, _, P = attend.entmax_attention(q, K, V, alpha, scale)
    B = np.linalg.norm(V, axis=1).max()
    for trial in range(5):
        keep = np.sort(rng.choice(400, 250, replace=False))
        o_sp, _, _ = attend.entmax_attention(q, K[keep], V[keep], alpha, scale)
        delta = attend.dropped_mass(P, keep)
        err = np.linalg.norm(o_sp - o_full, axis=1)
        assert np.all(err <= 2 * B * delta + 1e-12)


def test_output_is_p_times_v():
    rng = np.random.default_rng(42)
    q, K, V = _data(rng, 300, 24)
    o, _, P = attend.entmax_attention(q, K, V, 1.5, 0.3)
    np.testing.assert_allclose(o, P @ V, rtol=1e-12, atol=1e-12)


def test_softmax_special_cases():
    rng = np.random.default_rng(43)
    V = rng.standard_normal((10, 8))
    K = np.zeros((10, 8))
    q = rng.standard_normal((2, 8))
    np.testing.assert_allclose(attend.softmax_attention(q, K, V, 1.0), np.tile(V.mean(0), (2, 1)),
                               rtol=1e-13, atol=1e-13)
    K[3] = 1e3 * q[0]
    o = attend.softmax_attention(q[:1], K, V, 1.0)
    np.testing.assert_allclose(o[0], V[3], atol=1e-12)


def test_two_token_sparsemax():
    V = np.array([[1.0, 0.0], [0.0, 1.0]])
    for a, b in [(0.2, 0.0), (0.0, 0.9), (3.0, 0.0)]:
        K = np.array([[a], [b]])
        q = np.array([[1.0]])
        o, _, _ = attend.entmax_attention(q, K, V, 2.0, 1.0)
        p1 = min(1.0, max(0.0, (a - b + 1.0) / 2.0))
        np.testing.assert_allclose(o[0], [p1, 1.0 - p1], atol=1e-14)


def test_token_indices_ragged():
    assert list(attend.token_indices([2, 0], 37, 16)) == list(range(0, 16)) + list(range(32, 37))


def test_subset_softmax_is_the_renormalised_restriction():
    rng = np.random.default_rng(44)
    q, K, V = _data(rng, 200, 16)
    scale = 0.4
    s = scale * (q @ K.T)                                   # [G, n]
    p_full = np.exp(s - s.max(axis=1, keepdims=True))
    p_full /= p_full.sum(axis=1, keepdims=True)
    o_full = attend.softmax_attention(q, K, V, scale)
    B = np.linalg.norm(V, axis=1).max()
    for trial in range(4):
        keep = np.sort(rng.choice(200, 60 + 30 * trial, replace=False))
        o_sub = attend.softmax_attention(q, K[keep], V[keep], scale)
        w = p_full[:, keep] / p_full[:, keep].sum(axis=1, keepdims=True)
        np.testing.assert_allclose(o_sub, w @ V[keep], rtol=1e-10, atol=1e-12)
        delta = attend.dropped_mass(p_full, keep)
        assert np.all(delta > 0)
        err = np.linalg.norm(o_sub - o_full, axis=1)
        assert np.all(err <= 2 * B * delta + 1e-12)


def test_two_token_entmax_15_closed_form():
    """alpha = 1.5 over two tokens, solved by hand on x = (alpha - 1) * scale * q.k:
    both tokens carry weight iff |x1 - x2| < 1, and then (x1 - tau)^2 + (x2 - tau)^2 = 1
    gives tau = ((x1 + x2) - sqrt(2 - (x1 - x2)^2)) / 2 and p_i = (x_i - tau)^2.
    Pins the (alpha - 1) factor of the entmax input (alpha = 2 cannot)."""
    V = np.array([[1.0, 0.0], [0.0, 1.0]])
    q = np.array([[1.0]])
    for s1, s2, scale in [(1.0, 0.0, 1.0), (0.3, 1.1, 1.0), (2.5, 0.0, 1.0), (4.0, 1.0, 0.5), (0.0, 0.0, 1.0)]:
        x1, x2 = 0.5 * scale * s1, 0.5 * scale * s2
        if abs(x1 - x2) < 1.0:
            tau = ((x1 + x2) - np.sqrt(2.0 - (x1 - x2) ** 2)) / 2.0
            p = [(x1 - tau) ** 2, (x2 - tau) ** 2]
        else:
            p = [1.0, 0.0] if x1 > x2 else [0.0, 1.0]
        o, _, _ = attend.entmax_attention(q, np.array([[s1], [s2]]), V, 1.5, scale)
        np.testing.assert_allclose(o[0], p, atol=1e-13)
