"""The oracle's pins catch plausible mistakes: each case plants one mistake in
the oracle (in memory, on the CPU, through monkeypatch) and checks that a named
pin then fails.  The pins are the ones in tests/test_oracle_*.py; a pin that
stayed green under its mistake would leave that part of the oracle unchecked.
"""
import math

import numpy as np
import pytest
from scipy.special import ndtr

import test_oracle_attend as TA
import test_oracle_entmax as TE
import test_oracle_gauss as TG
import test_oracle_pages as TP
import test_oracle_select as TS
from oracle import attend, entmax, gauss, pages, select

_tau_sort, _probs, _meta = entmax.tau_sort, entmax.probs, pages.page_metadata
_attention, _softmax, _g, _F = attend.entmax_attention, attend.softmax_attention, gauss.g, gauss.F


def _prefix_taus(x, alpha, root_sign=-1.0):
    x = np.asarray(x, dtype=np.float64).ravel()
    z = np.sort(x[np.isfinite(x)])[::-1]
    k = np.arange(1, z.size + 1, dtype=np.float64)
    cs = np.cumsum(z)
    if alpha == 2.0:
        tk = (cs - 1.0) / k
        return z, tk, tk < z
    mean, msq = cs / k, np.cumsum(z * z) / k
    disc = mean * mean - msq + 1.0 / k
    ok = disc >= 0
    tk = np.where(ok, mean + root_sign * np.sqrt(np.where(ok, disc, 0.0)), np.inf)
    return z, tk, ok & (tk < z)


def larger_root(x, alpha):
    if alpha != 1.5:
        return _tau_sort(x, alpha)
    z, tk, ok = _prefix_taus(x, alpha, +1.0)
    idx = np.nonzero(ok)[0]
    return float(tk[idx[-1]]) if idx.size else float(z[0] - 1.0)


def first_prefix(x, alpha):
    _, tk, ok = _prefix_taus(x, alpha)
    return float(tk[np.nonzero(ok)[0][0]])


def power_alpha_minus_one(x, alpha, method="sort"):
    _, tau = _probs(x, alpha, method)
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(invalid="ignore"):
        return np.where(np.isfinite(x), np.maximum(x - tau, 0.0), 0.0) ** (alpha - 1.0), tau


def bound_min(q, kmin, kmax, scale):
    q = np.asarray(q, dtype=np.float64)
    lo, hi = q[:, None, :] * np.asarray(kmin)[None], q[:, None, :] * np.asarray(kmax)[None]
    return scale * np.minimum(lo, hi).sum(axis=2)


def bound_kmax_only(q, kmin, kmax, scale):
    return scale * (np.asarray(q, dtype=np.float64)[:, None, :] * np.asarray(kmax)[None]).sum(axis=2)


def sample_variance(keys, ps):
    out = _meta(keys, ps)
    keys = np.asarray(keys, dtype=np.float64)
    for p in range(len(out["count"])):
        blk = keys[p * ps:(p + 1) * ps]
        out["var"][p] = blk.var(axis=0, ddof=1) if blk.shape[0] > 1 else 0.0
    return out


def count_always_ps(keys, ps):
    out = _meta(keys, ps)
    out["count"][:] = ps
    return out


def v_scaled_once(q, mean, var, scale):
    q = np.asarray(q, dtype=np.float64)
    return scale * (q @ np.asarray(mean).T), scale * ((q * q) @ np.asarray(var).T)


def v_with_abs_q(q, mean, var, scale):
    q = np.asarray(q, dtype=np.float64)
    return scale * (q @ np.asarray(mean).T), scale * scale * (np.abs(q) @ np.asarray(var).T)


def ties_to_higher_index(keys, k):
    keys = np.asarray(keys, dtype=np.float32)
    order = sorted(range(keys.size), key=lambda i: (-float(keys[i]), -i))
    return np.array(sorted(order[:min(int(k), keys.size)]), dtype=np.int64)


def unsorted_selection(keys, k):
    keys = np.asarray(keys, dtype=np.float32)
    order = sorted(range(keys.size), key=lambda i: (-float(keys[i]), i))
    return np.array(order[:min(int(k), keys.size)], dtype=np.int64)


def budget_floor(P, budget, frac):
    k = int(budget) if budget >= 0 else int(math.floor(float(np.float32(frac)) * float(P)))
    return max(0, min(k, int(P)))


def _keep(est, tau_hat, alpha, delta, cmp, reduce, am1=True):
    est = np.asarray(est, dtype=np.float32)
    tau_hat = np.asarray(tau_hat, dtype=np.float32)
    lhs = (np.float32(alpha - 1.0) * est).astype(np.float32) if am1 else est
    rhs = (tau_hat - np.float32(delta)).astype(np.float32)
    return np.nonzero(reduce(cmp(lhs, rhs[:, None]), axis=0))[0].astype(np.int64)


def keep_delta_sign(est, tau_hat, alpha, delta):
    return _keep(est, tau_hat, alpha, -delta, np.greater_equal, np.any)


def keep_without_alpha(est, tau_hat, alpha, delta):
    return _keep(est, tau_hat, alpha, delta, np.greater_equal, np.any, am1=False)


def keep_strict(est, tau_hat, alpha, delta):
    return _keep(est, tau_hat, alpha, delta, np.greater, np.any)


def keep_all_heads(est, tau_hat, alpha, delta):
    return _keep(est, tau_hat, alpha, delta, np.greater_equal, np.all)


def x_without_alpha(q, K, V, alpha, scale, method="sort"):
    return _attention(q, K, V, alpha, scale / (alpha - 1.0), method)


def softmax_unscaled(q, K, V, scale):
    return _softmax(q, K, V, 1.0)


def drops_partial_page(pages_, seq_len, ps):
    return np.asarray([t for p in sorted(int(x) for x in pages_) if (p + 1) * ps <= seq_len
                       for t in range(p * ps, (p + 1) * ps)], dtype=np.int64)


def kept_mass(p_full, kept):
    keep = np.zeros(p_full.shape[-1], dtype=bool)
    keep[kept] = True
    return p_full[..., keep].sum(axis=-1)


def z_without_root(ps):
    return np.array([0.0, 0.0] + [2.0 * math.log(n) for n in range(2, ps + 1)])


def z_half_log(ps):
    return np.array([0.0, 0.0] + [math.sqrt(math.log(n)) for n in range(2, ps + 1)])


def est_with_variance(m, v, n, ps):
    return np.asarray(m, dtype=np.float64) + np.maximum(v, 0.0) * gauss.z_table(ps)[np.asarray(n)]


def est_z_off_by_one(m, v, n, ps):
    z = gauss.z_table(ps)
    return np.asarray(m, dtype=np.float64) + np.sqrt(np.maximum(v, 0.0)) * z[np.maximum(np.asarray(n) - 1, 0)]


def _gauss_closed(mp, sp, tau, alpha, method, form):
    if method != "closed" or alpha not in form:
        return _g(mp, sp, tau, alpha, method)
    mp, sp = np.asarray(mp, dtype=np.float64), np.asarray(sp, dtype=np.float64)
    u = mp - tau
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(sp > 0, u / np.where(sp > 0, sp, 1.0), 0.0)
    phi = np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)
    return np.where(sp > 0, form[alpha](u, sp, z, phi), np.maximum(u, 0.0) ** (1.0 / (alpha - 1.0)))


def g15_without_spread_term(mp, sp, tau, alpha, method="closed"):
    return _gauss_closed(mp, sp, tau, alpha, method, {1.5: lambda u, s, z, phi: u * u * ndtr(z) + u * s * phi})


def g2_without_density_term(mp, sp, tau, alpha, method="closed"):
    return _gauss_closed(mp, sp, tau, alpha, method, {2.0: lambda u, s, z, phi: u * ndtr(z)})


def F_one_token_per_page(tau, m, v, n, alpha):
    return _F(tau, m, v, np.ones_like(np.asarray(n)), alpha)


def F_spread_without_alpha(tau, m, v, n, alpha):
    mp, sp = (alpha - 1.0) * np.asarray(m, dtype=np.float64), np.sqrt(np.maximum(np.asarray(v, dtype=np.float64), 0))
    return float(np.sum(np.asarray(n, dtype=np.float64) * gauss.g(mp, sp, tau, alpha)))


def F_variance_for_std(tau, m, v, n, alpha):
    am1 = alpha - 1.0
    mp, sp = am1 * np.asarray(m, dtype=np.float64), am1 * np.maximum(np.asarray(v, dtype=np.float64), 0)
    return float(np.sum(np.asarray(n, dtype=np.float64) * gauss.g(mp, sp, tau, alpha)))


# (planted mistake, oracle function replaced, pin that must fail)
CASES = [
    ("1.5-entmax takes the larger root", entmax, "tau_sort", larger_root,
     lambda: TE.test_sort_and_bisect_agree(1.5)),
    ("sorted prefix: first consistent k", entmax, "tau_sort", first_prefix,
     lambda: TE.test_sort_and_bisect_agree(2.0)),
    ("weights raised to alpha - 1", entmax, "probs", power_alpha_minus_one,
     lambda: TE.test_simplex_and_shift(3.0)),
    ("bound takes the min", pages, "bbox_bound", bound_min,
     lambda: TP.test_bound_dominates_every_score(16, 64)),
    ("bound ignores the sign of q", pages, "bbox_bound", bound_kmax_only, TP.test_bound_attained_on_corner),
    ("sample variance", pages, "page_metadata", sample_variance, TP.test_moments_invariants),
    ("every page counted full", pages, "page_metadata", count_always_ps, TP.test_moments_invariants),
    ("v scaled once", pages, "gauss_scores", v_scaled_once,
     TP.test_gauss_scores_are_the_score_moments_when_keys_vary_in_one_coordinate),
    ("v with |q|", pages, "gauss_scores", v_with_abs_q,
     TP.test_gauss_scores_are_the_score_moments_when_keys_vary_in_one_coordinate),
    ("top-k ties to the higher index", select, "topk", ties_to_higher_index,
     TS.test_signed_zero_ties_go_to_lower_index),
    ("top-k not sorted by page", select, "topk", unsorted_selection, TS.test_topk_random_and_planted),
    ("budget rounded down", select, "budget_pages", budget_floor, lambda: TS.test_budget_fraction(100, 1 / 16, 7)),
    ("margin added instead of subtracted", select, "gauss_keep", keep_delta_sign,
     TS.test_gauss_keep_threshold_is_inclusive_and_a_union_over_the_group),
    ("keep rule without alpha - 1", select, "gauss_keep", keep_without_alpha, TS.test_gauss_keep_degenerate_cases),
    ("keep rule strict", select, "gauss_keep", keep_strict,
     TS.test_gauss_keep_threshold_is_inclusive_and_a_union_over_the_group),
    ("keep rule needs every head", select, "gauss_keep", keep_all_heads,
     TS.test_gauss_keep_threshold_is_inclusive_and_a_union_over_the_group),
    ("entmax input without alpha - 1", attend, "entmax_attention", x_without_alpha,
     TA.test_two_token_entmax_15_closed_form),
    ("softmax without the scale", attend, "softmax_attention", softmax_unscaled,
     TA.test_subset_softmax_is_the_renormalised_restriction),
    ("partial last page dropped", attend, "token_indices", drops_partial_page, TA.test_token_indices_ragged),
    ("delta counts the kept mass", attend, "dropped_mass", kept_mass,
     lambda: TA.test_support_recovery_is_bitwise_exact(1.5)),
    ("z_n without the square root", gauss, "z_table", z_without_root,
     TG.test_z_bounds_the_expected_maximum_of_n_normals),
    ("z_n = sqrt(ln n)", gauss, "z_table", z_half_log,
     TG.test_z_bounds_the_expected_maximum_of_n_normals),
    ("page maximum from the variance", gauss, "est_max", est_with_variance,
     TP.test_estimated_page_maximum_scales_with_the_spread),
    ("page maximum with z of n - 1", gauss, "est_max", est_z_off_by_one,
     TP.test_estimated_page_maximum_scales_with_the_spread),
    ("E[(X-t)_+^2] without the spread term", gauss, "g", g15_without_spread_term,
     lambda: TG.test_g_against_monte_carlo(1.5)),
    ("E[(X-t)_+] without the density term", gauss, "g", g2_without_density_term,
     lambda: TG.test_g_against_quadrature(2.0)),
    ("F ignores tokens per page", gauss, "F", F_one_token_per_page,
     lambda: TG.test_pages_of_equal_tokens_reduce_to_exact_entmax_of_the_multiset(1.5)),
    ("F spread without alpha - 1", gauss, "F", F_spread_without_alpha,
     lambda: TG.test_F_is_the_expected_mass_of_the_page_draws(1.5)),
    ("F uses the variance as the spread", gauss, "F", F_variance_for_std,
     lambda: TG.test_F_is_the_expected_mass_of_the_page_draws(2.0)),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_pin_catches_planted_mistake(case, monkeypatch):
    _, module, name, mistake, pin = case
    pin()                                   # green on the oracle as it is
    monkeypatch.setattr(module, name, mistake)
    with pytest.raises(AssertionError):
        pin()
