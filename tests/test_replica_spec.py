"""The fp32 replicas follow the operation order entmaxkv.h states, bit for bit.

Page selection is decided on fp32 values, so the library and the oracle's
replicas must compute them in one stated order (the header comment of
entmaxkv_append_metadata and entmaxkv_score_pages).  The GPU parity tests show
the library equals the C replicas bit for bit; this test shows the C replicas
equal a transcription of the header's text into exactly rounded fp32
arithmetic, so both follow the stated order and not merely each other.

Exact fp32 arithmetic here: a sum, product, quotient or square root of fp32
values computed in float64 and rounded once to fp32 is the correctly rounded
fp32 result (float64 carries more than 2 * 24 + 2 bits); a fused multiply-add
is rounded once from the exact rational value.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import replica

f32 = np.float32


def rn32(x):
    """Round an exact rational to the nearest fp32, ties to even (normal range)."""
    if x == 0:
        return f32(0.0)
    neg, a = x < 0, abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** (max(e, -126) - 23)
    m = a / ulp
    k = m.numerator // m.denominator
    rem = m - k
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and k % 2):
        k += 1
    v = f32(float(k * ulp))
    return -v if neg else v


def fma(a, b, c):
    return rn32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def add(a, b):
    return f32(np.float64(a) + np.float64(b))


def sub(a, b):
    return f32(np.float64(a) - np.float64(b))


def mul(a, b):
    return f32(np.float64(a) * np.float64(b))


def div(a, b):
    return f32(np.float64(a) / np.float64(b))


def sqrt(a):
    return f32(np.sqrt(np.float64(a)))


def dot8(terms_a, terms_b):
    """d cut into 8 consecutive slices, each a chain of fmas from 0 in
    ascending d, slice sums combined as ((S0+S1)+(S2+S3))+((S4+S5)+(S6+S7))."""
    d = len(terms_a)
    w = d // 8
    S = []
    for k in range(8):
        acc = f32(0.0)
        for j in range(k * w, (k + 1) * w):
            acc = fma(terms_a[j], terms_b[j], acc)
        S.append(acc)
    return add(add(add(S[0], S[1]), add(S[2], S[3])), add(add(S[4], S[5]), add(S[6], S[7])))


def meta_spec(keys, ps):
    """Header of entmaxkv_append_metadata: per page and coordinate in token
    order; first token mean = x, m2 = 0, kmin = kmax = x; a token with n tokens
    filled after it: d1 = x - mean; mean += d1 / n; m2 = fma(d1, x - mean, m2)."""
    L, d = keys.shape
    P = (L + ps - 1) // ps
    out = {k: np.zeros((P, d), np.float32) for k in ("kmin", "kmax", "mean", "m2")}
    for p in range(P):
        for j in range(d):
            for t in range(p * ps, min(L, (p + 1) * ps)):
                x = keys[t, j]
                if t == p * ps:
                    mean, m2, lo, hi = x, f32(0.0), x, x
                    continue
                n = f32(t - p * ps + 1)
                d1 = sub(x, mean)
                mean = add(mean, div(d1, n))
                m2 = fma(d1, sub(x, mean), m2)
                lo, hi = (x if x < lo else lo), (x if x > hi else hi)
            out["kmin"][p, j], out["kmax"][p, j], out["mean"][p, j], out["m2"][p, j] = lo, hi, mean, m2
    return out


def bound_spec(q, kmin, kmax, scale):
    """Header of entmaxkv_score_pages, BBOX: scale * sum_d q_d (q_d >= 0 ?
    kmax_d : kmin_d) per head, max over the group's heads, -0 -> +0."""
    G, P = q.shape[0], kmin.shape[0]
    ub = np.zeros((G, P), np.float32)
    for p in range(P):
        for h in range(G):
            sel = [kmax[p, j] if q[h, j] >= 0 else kmin[p, j] for j in range(q.shape[1])]
            ub[h, p] = mul(dot8(q[h], sel), scale)
    ubg = ub.max(axis=0)
    ubg[ubg == 0] = 0.0
    return ub, ubg


def gauss_spec(q, mean, m2, count, scale, z):
    """Header of entmaxkv_score_pages, GAUSS: m = scale * sum q_d mean_d,
    v = ((sum (q_d*q_d) m2_d) / n) * scale^2, est = fma(sqrt(v), z_n, m)."""
    G, P = q.shape[0], mean.shape[0]
    m, v, est = (np.zeros((G, P), np.float32) for _ in range(3))
    scale2 = mul(scale, scale)
    for h in range(G):
        q2 = [mul(x, x) for x in q[h]]
        for p in range(P):
            m[h, p] = mul(dot8(q[h], mean[p]), scale)
            v[h, p] = mul(div(dot8(q2, m2[p]), f32(count[p])), scale2)
            est[h, p] = fma(sqrt(v[h, p]), z[count[p]], m[h, p])
    return m, v, est


def test_exact_fma_rounds_once():
    a, b = f32(1.0 + 2.0 ** -12), f32(1.0 - 2.0 ** -12)
    c = f32(-1.0)
    assert fma(a, b, c) == f32(-(2.0 ** -24))          # exact: a*b - 1 = -2^-24
    assert rn32(Fraction(1) + Fraction(1, 2 ** 24)) == f32(1.0)                      # tie to even
    assert rn32(Fraction(1) + Fraction(3, 2 ** 25)) == f32(1.0 + 2.0 ** -23)         # above the tie


@pytest.mark.parametrize("d,ps", [(64, 16), (128, 16)])
def test_replicas_follow_the_header_order(d, ps):
    rng = np.random.default_rng(50)
    L = 3 * ps + 5                                          # three full pages and a ragged one
    keys = (rng.standard_normal((L, d)) * 0.7 + rng.standard_normal(d)).astype(np.float32)
    q = rng.standard_normal((4, d)).astype(np.float32)
    scale = f32(1.0 / np.sqrt(d))

    spec = meta_spec(keys, ps)
    rep = replica.page_meta(keys, ps)
    for k in ("kmin", "kmax", "mean", "m2"):
        assert np.array_equal(rep[k].view(np.uint32), spec[k].view(np.uint32)), k

    ub_s, ubg_s = bound_spec(q, spec["kmin"], spec["kmax"], scale)
    ub_r, ubg_r = replica.bound(q, rep["kmin"], rep["kmax"], float(scale))
    assert np.array_equal(ub_r.view(np.uint32), ub_s.view(np.uint32))
    assert np.array_equal(ubg_r.view(np.uint32), ubg_s.view(np.uint32))

    z = replica.z_table_f32(ps)
    ms, vs, es = gauss_spec(q, spec["mean"], spec["m2"], rep["count"], scale, z)
    mr, vr, er = replica.gauss(q, rep["mean"], rep["m2"], rep["count"], float(scale), ps)
    for a, b in ((mr, ms), (vr, vs), (er, es)):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_header_order_differs_from_a_serial_sum():
    """The stated order is not a formality: a single serial fma chain over d
    gives a different fp32 bound for some pages of the same data."""
    rng = np.random.default_rng(51)
    d = 128
    kmin = rng.standard_normal((40, d)).astype(np.float32)
    kmax = (kmin + np.abs(rng.standard_normal((40, d)))).astype(np.float32)
    q = rng.standard_normal((1, d)).astype(np.float32)
    ub, _ = bound_spec(q, kmin, kmax, f32(1.0))
    serial = []
    for p in range(40):
        acc = f32(0.0)
        for j in range(d):
            acc = fma(q[0, j], kmax[p, j] if q[0, j] >= 0 else kmin[p, j], acc)
        serial.append(acc)
    assert np.any(np.array(serial, np.float32).view(np.uint32) != ub[0].view(np.uint32))
