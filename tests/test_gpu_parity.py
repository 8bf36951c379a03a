"""GPU parity of every step of the decode path against the CPU oracle.

Every call goes through the C ABI (sparse_long_context_min_b200.binding).
Sizes span several pipeline stages, several splits and a ragged last page;
the oracle side is computed from the generator's tensors only.
"""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

import helpers as H
from oracle import attend, gauss, select
from sparse_long_context_min_b200 import binding as B
from sparse_long_context_min_b200 import workloads
from sparse_long_context_min_b200.step import DecodeStep, build_pool

pytestmark = pytest.mark.gpu


def _wl(n, lengths=None, B_=None, **kw):
    cfg = workloads.config(n, B=B_)
    if lengths is not None:
        cfg = replace(cfg, B=len(lengths), lengths=list(lengths))
    if kw:
        cfg = replace(cfg, **kw)
    return workloads.Workload(cfg, device="cuda")


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _assert_ok(st):
    torch.cuda.synchronize()
    assert int(st.item()) == 0, B.status_string(int(st.item()))


# (config, lengths) cases: fp32 tiny, bf16 d=128 ps=64 with ragged pages, permuted pool
CASES = {
    "tiny": (1, [4096 + 5]),
    "llama": (2, [16384 + 1]),
    "ragged": (5, [5000, 12345, 777]),
}


@pytest.fixture(scope="module", params=list(CASES))
def built(request):
    n, lens = CASES[request.param]
    wl = _wl(n, lens)
    pool, seq_lens = build_pool(wl)
    oseqs = [H.OracleSeq(wl, b) for b in range(wl.cfg.B)]
    return wl, pool, seq_lens, oseqs


def test_append_metadata_bitexact(built):
    wl, pool, seq_lens, oseqs = built
    cfg = wl.cfg
    assert seq_lens.cpu().tolist() == cfg.lengths
    pt = wl.page_table.cpu()
    for b, o in enumerate(oseqs):
        P = cfg.pages(b)
        phys = pt[b, :P].long()
        for g in range(cfg.H_kv):
            m = o.meta(g)
            assert np.array_equal(pool.kmin[phys, g].float().cpu().numpy(), m["kmin"])
            assert np.array_equal(pool.kmax[phys, g].float().cpu().numpy(), m["kmax"])
            assert np.array_equal(pool.mean[phys, g].cpu().numpy(), m["mean"])
            assert np.array_equal(pool.m2[phys, g].cpu().numpy(), m["m2"])
            # pool contents are the appended tokens
            kp = pool.k_pool[phys, g].float().cpu().numpy().reshape(P * cfg.ps, cfg.d)[:o.L]
            assert np.array_equal(kp, o.keys[g])
        assert np.array_equal(pool.count[phys].cpu().numpy(), o.meta(0)["count"])


def test_append_one_token_at_a_time_matches_whole_pages():
    wl = _wl(2, [200])
    cfg = wl.cfg
    pool_a, _ = build_pool(wl)
    pool_b = B.Pool.allocate(wl.num_phys, cfg.H_kv, cfg.ps, cfg.d, cfg.dtype)
    seq = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = _status()
    k, v = wl.sequence(0)
    pt = wl.page_table
    for t in range(0, 200, 7):            # chunks of 7 tokens cross page boundaries
        kk = k[:, t:t + 7].unsqueeze(0).contiguous()
        vv = v[:, t:t + 7].unsqueeze(0).contiguous()
        B.append_metadata(pool_b, kk, vv, pt, seq, st)
    _assert_ok(st)
    assert int(seq.item()) == 200
    for name in ("kmin", "kmax", "mean", "m2", "count", "k_pool", "v_pool"):
        a, b_ = getattr(pool_a, name), getattr(pool_b, name)
        assert torch.equal(a, b_), name


@pytest.mark.parametrize("n_new", [1, 5, 64])
def test_append_score_equals_append_then_score(n_new):
    """entmaxkv_append_score_pages (the append folded into the scoring launch)
    leaves exactly what entmaxkv_append_metadata followed by
    entmaxkv_score_pages(BBOX) leaves: pool rows, metadata, counts, lengths and
    bounds, bit for bit, over appends that fill, cross and start pages of a
    ragged batch with permuted physical pages."""
    wl = _wl(5, [5000, 12345 - 12, 777, 64 * 9], decode_steps=8 * 64)
    cfg = wl.cfg
    pool_a, lens_a = build_pool(wl)
    pool_b, lens_b = build_pool(wl)
    st = _status()
    ub_a = torch.empty(cfg.B, cfg.H_kv, wl.max_pages, device="cuda")
    ub_b = torch.empty_like(ub_a)
    scale = H.scale32(cfg)
    for t in range(4):
        g = torch.Generator(device="cuda").manual_seed(100 + t)
        k = torch.randn(cfg.B, cfg.H_kv, n_new, cfg.d, generator=g, device="cuda").to(cfg.dtype)
        v = torch.randn(cfg.B, cfg.H_kv, n_new, cfg.d, generator=g, device="cuda").to(cfg.dtype)
        q = torch.randn(cfg.B, cfg.H_q, cfg.d, generator=g, device="cuda")
        B.append_metadata(pool_a, k, v, wl.page_table, lens_a, st)
        B.score_pages(pool_a, q, wl.page_table, lens_a, B.SCORE_BBOX, scale, st, ub=ub_a)
        B.append_score_pages(pool_b, k, v, q, wl.page_table, lens_b, scale, st, ub_b)
        _assert_ok(st)
        assert torch.equal(lens_a, lens_b)
        for name in ("kmin", "kmax", "mean", "m2", "count", "k_pool", "v_pool"):
            assert torch.equal(getattr(pool_a, name), getattr(pool_b, name)), (t, name)
        for b in range(cfg.B):
            P = (int(lens_a[b]) + cfg.ps - 1) // cfg.ps
            assert torch.equal(ub_a[b, :, :P], ub_b[b, :, :P]), (t, b)
            assert bool(torch.all(ub_b[b, :, P:] == -float("inf")))


def test_score_bbox_bitexact(built):
    wl, pool, seq_lens, oseqs = built
    cfg = wl.cfg
    st = _status()
    ub = torch.empty(cfg.B, cfg.H_kv, wl.max_pages, device="cuda")
    B.score_pages(pool, wl.q, wl.page_table, seq_lens, B.SCORE_BBOX, H.scale32(cfg), st, ub=ub)
    _assert_ok(st)
    ub = ub.cpu().numpy()
    for b, o in enumerate(oseqs):
        P = cfg.pages(b)
        for g in range(cfg.H_kv):
            assert np.array_equal(ub[b, g, :P], o.ubg(g)), (b, g)
            assert np.all(ub[b, g, P:] == -np.inf)


@pytest.mark.parametrize("frac", [1 / 32, 1 / 8])
def test_topk_selection_bitexact(built, frac):
    wl, pool, seq_lens, oseqs = built
    cfg = wl.cfg
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=frac, alpha=cfg.alpha)
    step.score(wl.q)
    step.choose()
    step.check()
    sel, cnt = step.sel.cpu().numpy(), step.sel_count.cpu().numpy()
    for b, o in enumerate(oseqs):
        for g in range(cfg.H_kv):
            ref = o.topk(g, -1, frac)
            assert cnt[b, g] == len(ref)
            assert np.array_equal(sel[b, g, :cnt[b, g]], ref), (b, g)


def test_topk_ties_signed_zeros_and_budgets():
    """select() on a hand-made bound array with heavy ties, +-0 and every budget regime."""
    rng = np.random.default_rng(7)
    P, Bn, Hkv = 3000, 3, 2
    vals = np.array([-1.0, -0.0, 0.0, 0.25, 0.25, 2.0, 5.5], dtype=np.float32)
    ub = vals[rng.integers(0, len(vals), (Bn, Hkv, P))]
    ub[1, 1] = rng.standard_normal(P).astype(np.float32)
    ub[2] = 0.25                                  # all equal
    seq_lens = torch.tensor([P * 16, P * 16 - 15, 40 * 16], dtype=torch.int32, device="cuda")
    for budget in (0, 1, 7, 300, 2999, 3000, 5000):
        k_max = max(1, budget)
        sel = torch.full((Bn, Hkv, k_max), -7, dtype=torch.int32, device="cuda")
        cnt = torch.empty(Bn, Hkv, dtype=torch.int32, device="cuda")
        st = _status()
        B.select(B.SELECT_TOPK, seq_lens, 16, Hkv * 4, Hkv, P, k_max, sel, cnt, st,
                 ub=torch.from_numpy(ub).cuda(), budget=budget)
        _assert_ok(st)
        for b in range(Bn):
            Pb = (int(seq_lens[b]) + 15) // 16
            for g in range(Hkv):
                ref = select.topk(ub[b, g, :Pb], select.budget_pages(Pb, budget, 0.0))
                c = int(cnt[b, g])
                assert c == len(ref)
                assert np.array_equal(sel[b, g, :c].cpu().numpy(), ref), (budget, b, g)


# bf16 cache shapes besides the benchmark's (G = 4, d = 128, pages of 64):
# one, two and eight query heads per kv head, d = 64, pages of 16
SHAPES = {
    "g1_d64_ps16": dict(H_q=8, H_kv=8, d=64, ps=16),
    "g2_d64_ps16": dict(H_q=16, H_kv=8, d=64, ps=16),
    "g8_d128_ps64": dict(H_q=64, H_kv=8, d=128, ps=64),
    "g4_d64_ps64": dict(H_q=32, H_kv=8, d=64, ps=64),
    "g8_d64_ps16": dict(H_q=32, H_kv=4, d=64, ps=16),
    "g2_d128_ps16": dict(H_q=8, H_kv=4, d=128, ps=16),
}


# fp32 caches take the streaming scoring kernel and the CUDA-core attention
FP32_SHAPES = {
    "f32_g8_d128_ps64": dict(H_q=64, H_kv=8, d=128, ps=64),
    "f32_g2_d128_ps16": dict(H_q=8, H_kv=4, d=128, ps=16),
}


@pytest.mark.parametrize("shape", list(SHAPES) + list(FP32_SHAPES))
def test_head_and_page_shapes(shape):
    if shape in FP32_SHAPES:
        wl = _wl(1, [3001, 1234], **FP32_SHAPES[shape])
    else:
        wl = _wl(2, [3001, 1234], **SHAPES[shape])
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 8, alpha=cfg.alpha)
    step.score(wl.q)
    step.choose()
    step.attend(wl.q)
    step.check()
    ub, sel, cnt = step.ub.cpu().numpy(), step.sel.cpu().numpy(), step.sel_count.cpu().numpy()
    out = step.out.cpu().numpy()
    # the Gaussian page model of the same shape (role-split moments kernel where the layout allows)
    st = _status()
    gshape = (cfg.B, cfg.H_q, wl.max_pages)
    gm, gv, ge = (torch.empty(gshape, device="cuda") for _ in range(3))
    B.score_pages(pool, wl.q, wl.page_table, seq_lens, B.SCORE_GAUSS, H.scale32(cfg), st, m=gm, v=gv, est_max=ge)
    _assert_ok(st)
    gm, gv, ge = gm.cpu().numpy(), gv.cpu().numpy(), ge.cpu().numpy()
    G = cfg.G
    for b in range(cfg.B):
        o = H.OracleSeq(wl, b)
        P = cfg.pages(b)
        for g in range(cfg.H_kv):
            rm, rv, re = o.gauss(g)
            sl = slice(g * G, (g + 1) * G)
            assert np.array_equal(gm[b, sl, :P], rm) and np.array_equal(gv[b, sl, :P], rv), (b, g)
            assert np.array_equal(ge[b, sl, :P], re) and np.all(ge[b, sl, P:] == -np.inf), (b, g)
            assert np.array_equal(ub[b, g, :P], o.ubg(g)), (b, g)
            ref = o.topk(g, -1, 1 / 8)
            assert np.array_equal(sel[b, g, :cnt[b, g]], ref), (b, g)
            o_ref, _ = o.attention(g, ref, cfg.alpha)
            H.compare_out(out[b, g * G:(g + 1) * G], o_ref, cfg.dtype)


def _topk_cases():
    rng = np.random.default_rng(11)
    big_tie = np.full(5000, 0.25, np.float32)
    big_tie[rng.permutation(5000)[:100]] = 1.0          # threshold inside > 1024 equal keys
    outlier = rng.random(5000).astype(np.float32)
    outlier[17] = 1e6                                    # first bucket map squeezes the rest into one bucket
    dense = (1.0 + np.arange(3000, dtype=np.float32) * np.float32(2.0 ** -22)).astype(np.float32)
    dense[5] = -1e30
    rng.shuffle(dense)                                   # 3000 distinct keys a few ulps apart
    mid = rng.standard_normal(20000).astype(np.float32)  # 20 keys per thread of the one-CTA kernel
    infs = rng.standard_normal(9000).astype(np.float32)
    infs[rng.permutation(9000)[:2000]] = -np.inf         # empty pages bound at -inf
    infs[rng.permutation(9000)[:5]] = np.inf
    wide = rng.standard_normal(60000).astype(np.float32) # several keys per thread of an 8-CTA cluster
    huge = rng.standard_normal(70001).astype(np.float32) # past the cluster kernel: global-memory top-k
    huge[rng.permutation(70001)[:3000]] = 0.5            # with a large tie
    huge[rng.permutation(70001)[:500]] = -np.inf         # and empty pages
    return {"big_tie": big_tie, "outlier": outlier, "dense": dense, "mid": mid, "infs": infs, "wide": wide,
            "huge": huge}


@pytest.mark.parametrize("case", ["big_tie", "outlier", "dense", "mid", "infs", "wide", "huge"])
def test_topk_narrowing_rounds(case):
    """Key sets whose threshold bucket holds more than the exact-rank capacity,
    so the selection narrows over several rounds (or ends in a tie round)."""
    keys = _topk_cases()[case]
    P = len(keys)
    ub = torch.from_numpy(keys).reshape(1, 1, P).cuda()
    seq_lens = torch.tensor([P * 16], dtype=torch.int32, device="cuda")
    for budget in (1, 300, 2500, P - 1):
        sel = torch.full((1, 1, budget), -7, dtype=torch.int32, device="cuda")
        cnt = torch.empty(1, 1, dtype=torch.int32, device="cuda")
        st = _status()
        B.select(B.SELECT_TOPK, seq_lens, 16, 4, 1, P, budget, sel, cnt, st, ub=ub, budget=budget)
        _assert_ok(st)
        ref = select.topk(keys, budget)
        assert int(cnt[0, 0]) == len(ref)
        assert np.array_equal(sel[0, 0].cpu().numpy()[:len(ref)], ref), (case, budget)


def test_score_gauss_bitexact(built):
    wl, pool, seq_lens, oseqs = built
    cfg = wl.cfg
    st = _status()
    shape = (cfg.B, cfg.H_q, wl.max_pages)
    m = torch.empty(shape, device="cuda")
    v = torch.empty(shape, device="cuda")
    e = torch.empty(shape, device="cuda")
    B.score_pages(pool, wl.q, wl.page_table, seq_lens, B.SCORE_GAUSS, H.scale32(cfg), st, m=m, v=v, est_max=e)
    _assert_ok(st)
    m, v, e = m.cpu().numpy(), v.cpu().numpy(), e.cpu().numpy()
    G = cfg.G
    for b, o in enumerate(oseqs):
        P = cfg.pages(b)
        for g in range(cfg.H_kv):
            rm, rv, re = o.gauss(g)
            sl = slice(g * G, (g + 1) * G)
            assert np.array_equal(m[b, sl, :P], rm)
            assert np.array_equal(v[b, sl, :P], rv)
            assert np.array_equal(e[b, sl, :P], re)
            assert np.all(e[b, sl, P:] == -np.inf)


def _check_gauss_head(o, g, got, alpha, delta, kept, iters=100):
    """Gaussian selection of one kv head against the oracle.

    got: the GPU's tau_hat of the group's query heads.  tau_hat must lie within
    its tolerance of the oracle's float64 root; the kept set must equal, bit for
    bit, the fp32 keep rule evaluated with the GPU's own threshold (the page
    estimates are bit-equal to the replica's, so only the threshold can differ);
    against the oracle's threshold, decisions may differ only inside the band the
    threshold's error spans.  Returns the number of such in-band differences."""
    G = o.cfg.G
    m, v, est = o.gauss(g)
    n = o.meta(g)["count"]
    ref = np.array([gauss.tau_hat(m[h].astype(np.float64), v[h].astype(np.float64), n, alpha, iters=iters)
                    for h in range(G)])
    got = np.asarray(got, dtype=np.float32)
    g64 = got.astype(np.float64)
    assert np.all(np.abs(g64 - ref) <= H.TAU_HAT_TOL * np.maximum(1.0, np.abs(ref))), (got, ref)
    assert np.array_equal(kept, select.gauss_keep(est, got, alpha, delta))
    band = np.abs(g64 - ref) + 1e-6 * np.maximum(1.0, np.abs(ref))
    must_keep, must_drop = select.gauss_keep_bands(est, ref, alpha, delta, band[:, None])
    own = select.gauss_keep(est, ref.astype(np.float32), alpha, delta)
    diff = set(own.tolist()) ^ set(kept.tolist())
    assert not (diff & (set(must_keep.tolist()) | set(must_drop.tolist())))
    return len(diff)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
@pytest.mark.parametrize("delta", [0.0, 0.5])
def test_gauss_selection(alpha, delta):
    """Config-3 keys (random-walk pages, planted support), two ragged
    sequences: tau_hat, the exact kept sets of every kv head, and the entmax
    attention over the GPU's kept pages against the oracle."""
    wl = _wl(3, [8192 + 20, 4096 + 1])
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "gauss", alpha=alpha, delta=delta)
    step(wl.q)
    step.check()
    tau_gpu = step.tau_hat.cpu().numpy()
    sel, cnt, out = step.sel.cpu().numpy(), step.sel_count.cpu().numpy(), step.out.cpu().numpy()
    G = cfg.G
    for b in range(cfg.B):
        o = H.OracleSeq(wl, b)
        for g in range(cfg.H_kv):
            kept = sel[b, g, :cnt[b, g]]
            _check_gauss_head(o, g, tau_gpu[b, g * G:(g + 1) * G], alpha, delta, kept)
            o_ref, _ = o.attention(g, kept, alpha)
            H.compare_out(out[b, g * G:(g + 1) * G], o_ref, cfg.dtype)


@pytest.mark.parametrize("alpha", [1.05, 1.1, 1.25, 3.0])
def test_gauss_selection_any_alpha(alpha):
    """alpha outside {1.5, 2}: tau_hat from the 32-node Gauss-Legendre
    expectations (placed on the integrand's peak, so powers up to 1/(alpha-1)
    = 20 keep their mass) against the oracle's adaptive quadrature, the exact
    kept sets, and the attention over the GPU's kept pages."""
    wl = _wl(3, [4096 + 33])
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    delta = 0.5
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "gauss", alpha=alpha, delta=delta)
    step(wl.q)
    step.check()
    tau_gpu = step.tau_hat.cpu().numpy()
    sel, cnt, out = step.sel.cpu().numpy(), step.sel_count.cpu().numpy(), step.out.cpu().numpy()
    G = cfg.G
    o = H.OracleSeq(wl, 0)
    for g in (0, 6):
        kept = sel[0, g, :cnt[0, g]]
        _check_gauss_head(o, g, tau_gpu[0, g * G:(g + 1) * G], alpha, delta, kept, iters=60)
        o_ref, _ = o.attention(g, kept, alpha)
        H.compare_out(out[0, g * G:(g + 1) * G], o_ref, cfg.dtype)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_gauss_selection_many_pages(alpha):
    """Synthetic page statistics for 40001 pages (more than a CTA's register
    share in the tau_hat solve and several keep tiles per CTA): tau_hat
    against the oracle, and the kept set equal to the fp32 keep rule
    evaluated with the GPU's own tau_hat."""
    rng = np.random.default_rng(31)
    P, G, ps, delta = 40001, 4, 16, 0.5
    m = (0.6 * rng.standard_normal((1, G, P))).astype(np.float32)
    v = (0.3 * rng.random((1, G, P)) ** 2).astype(np.float32)
    count = np.full(P, ps, dtype=np.int64)
    count[-1] = 7                                          # ragged last page
    z = gauss.z_table(ps).astype(np.float32)
    est = (m + np.sqrt(v) * z[count][None, None, :]).astype(np.float32)
    L = (P - 1) * ps + 7
    seq_lens = torch.tensor([L], dtype=torch.int32, device="cuda")
    sel = torch.full((1, 1, P), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, 1, dtype=torch.int32, device="cuda")
    tau_hat = torch.empty(1, G, device="cuda")
    st = _status()
    B.select(B.SELECT_GAUSS, seq_lens, ps, G, 1, P, P, sel, cnt, st, m=torch.from_numpy(m).cuda(),
             v=torch.from_numpy(v).cuda(), est_max=torch.from_numpy(est).cuda(), alpha=alpha, delta=delta,
             tau_hat=tau_hat)
    _assert_ok(st)
    got = tau_hat.cpu().numpy()[0].astype(np.float64)
    ref = np.array([gauss.tau_hat(m[0, h].astype(np.float64), v[0, h].astype(np.float64), count, alpha)
                    for h in range(G)])
    assert np.all(np.abs(got - ref) <= H.TAU_HAT_TOL * np.maximum(1.0, np.abs(ref))), (got, ref)
    kept = sel[0, 0, :int(cnt[0, 0])].cpu().numpy()
    assert np.array_equal(kept, select.gauss_keep(est[0], tau_hat.cpu().numpy()[0], alpha, delta))


def test_sparse_attend_against_oracle(built):
    wl, pool, seq_lens, oseqs = built
    cfg = wl.cfg
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 16, alpha=cfg.alpha)
    # selection from the oracle, handed to the GPU as input
    sel = torch.zeros_like(step.sel)
    cnt = torch.zeros_like(step.sel_count)
    refs = {}
    for b, o in enumerate(oseqs):
        for g in range(cfg.H_kv):
            pages = o.topk(g, -1, 1 / 16)
            # add a few low-bound pages so the set is not only the best ones
            P = cfg.pages(b)
            extra = [p for p in range(0, P, 7) if p not in set(pages)][:3]
            pages = np.array(sorted(set(pages.tolist()) | set(extra)))[:step.k_max]
            sel[b, g, :len(pages)] = torch.from_numpy(pages.astype(np.int32))
            cnt[b, g] = len(pages)
            refs[b, g] = o.attention(g, pages, cfg.alpha)
    st = _status()
    out = torch.empty_like(step.out)
    tau = torch.empty_like(step.tau)
    vp = torch.zeros(cfg.B, cfg.H_kv, dtype=torch.int32, device="cuda")
    B.sparse_attend(pool, wl.q, wl.page_table, seq_lens, sel, cnt, cfg.alpha, H.scale32(cfg), out,
                    step.workspace, st, tau_out=tau, v_pages=vp)
    _assert_ok(st)
    out, tau, vp = out.cpu().numpy(), tau.cpu().numpy(), vp.cpu().numpy()
    G = cfg.G
    for (b, g), (o_ref, t_ref) in refs.items():
        H.compare_out(out[b, g * G:(g + 1) * G], o_ref, cfg.dtype)
        assert np.all(np.abs(tau[b, g * G:(g + 1) * G] - t_ref) <= 1e-5 * np.maximum(1, np.abs(t_ref)))
        # value pages loaded = selected pages holding a token with p > 0 (within a band
        # for tokens whose score sits on the threshold)
        o = oseqs[b]
        pages = sel[b, g, :cnt[b, g]].cpu().numpy()
        tok = attend.token_indices(pages, o.L, cfg.ps)
        x = (cfg.alpha - 1) * (o.keys[g][tok] @ o.qgroup(g).astype(np.float64).T) / math.sqrt(cfg.d)
        page_of = tok // cfg.ps
        sure = set(page_of[np.any(x > t_ref[None, :] + 1e-4, axis=1)].tolist())
        maybe = set(page_of[np.any(x > t_ref[None, :] - 1e-4, axis=1)].tolist())
        assert len(sure) <= vp[b, g] <= len(maybe), (len(sure), vp[b, g], len(maybe))


def test_decode_step_end_to_end(built):
    """score -> select -> attend on the GPU against the oracle's own pipeline."""
    wl, pool, seq_lens, oseqs = built
    cfg = wl.cfg
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 16, alpha=cfg.alpha)
    step(wl.q)
    step.check()
    sel, cnt = step.sel.cpu().numpy(), step.sel_count.cpu().numpy()
    out = step.out.cpu().numpy()
    G = cfg.G
    for b, o in enumerate(oseqs):
        for g in range(cfg.H_kv):
            pages = o.topk(g, -1, 1 / 16)
            assert np.array_equal(sel[b, g, :cnt[b, g]], pages)
            o_ref, _ = o.attention(g, pages, cfg.alpha)
            H.compare_out(out[b, g * G:(g + 1) * G], o_ref, cfg.dtype)


def test_full_entmax_and_softmax(built):
    wl, pool, seq_lens, oseqs = built
    cfg = wl.cfg
    st = _status()
    out = torch.empty(cfg.B, cfg.H_q, cfg.d, device="cuda")
    tau = torch.empty(cfg.B, cfg.H_q, device="cuda")
    ws = torch.empty(B.workspace_size(B.OP_FULL_ENTMAX, cfg.B, cfg.H_q, cfg.H_kv, wl.max_pages, 0, cfg.ps,
                                      cfg.d), dtype=torch.uint8, device="cuda")
    B.full_entmax_decode(pool, wl.q, wl.page_table, seq_lens, cfg.alpha, H.scale32(cfg), out, ws, st, tau_out=tau)
    out_s = torch.empty_like(out)
    ws_s = torch.empty(B.workspace_size(B.OP_FULL_SOFTMAX, cfg.B, cfg.H_q, cfg.H_kv, wl.max_pages, 0, cfg.ps,
                                        cfg.d), dtype=torch.uint8, device="cuda")
    B.full_softmax_decode(pool, wl.q, wl.page_table, seq_lens, H.scale32(cfg), out_s, ws_s, st)
    _assert_ok(st)
    out, out_s = out.cpu().numpy(), out_s.cpu().numpy()
    G = cfg.G
    for b, o in enumerate(oseqs):
        P = cfg.pages(b)
        for g in range(cfg.H_kv):
            o_ref, _ = o.attention(g, np.arange(P), cfg.alpha)
            H.compare_out(out[b, g * G:(g + 1) * G], o_ref, cfg.dtype)
            s_ref = attend.softmax_attention(o.qgroup(g), o.keys[g], o.values[g], 1.0 / math.sqrt(cfg.d))
            H.compare_out(out_s[b, g * G:(g + 1) * G], s_ref, cfg.dtype)


@pytest.mark.parametrize("alpha", [1.25, 1.7, 3.0])
def test_any_alpha_sparse_and_full(built, alpha):
    """alpha outside {1.5, 2}: threshold by the safeguarded Newton solve,
    weights by powf; against the oracle's bisection threshold."""
    wl, pool, seq_lens, oseqs = built
    cfg = wl.cfg
    G = cfg.G
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 16, alpha=alpha)
    step.score(wl.q)
    step.choose()
    st = _status()
    out = torch.empty_like(step.out)
    tau = torch.empty_like(step.tau)
    B.sparse_attend(pool, wl.q, wl.page_table, seq_lens, step.sel, step.sel_count, alpha, H.scale32(cfg), out,
                    step.workspace, st, tau_out=tau)
    full = torch.empty_like(out)
    ws = torch.empty(B.workspace_size(B.OP_FULL_ENTMAX, cfg.B, cfg.H_q, cfg.H_kv, wl.max_pages, 0, cfg.ps,
                                      cfg.d), dtype=torch.uint8, device="cuda")
    B.full_entmax_decode(pool, wl.q, wl.page_table, seq_lens, alpha, H.scale32(cfg), full, ws, st)
    _assert_ok(st)
    sel, cnt = step.sel.cpu().numpy(), step.sel_count.cpu().numpy()
    out, tau, full = out.cpu().numpy(), tau.cpu().numpy(), full.cpu().numpy()
    for b, o in enumerate(oseqs):
        for g in range(cfg.H_kv)[:3]:
            pages = sel[b, g, :cnt[b, g]]
            o_ref, t_ref = o.attention(g, pages, alpha)
            H.compare_out(out[b, g * G:(g + 1) * G], o_ref, cfg.dtype)
            assert np.all(np.abs(tau[b, g * G:(g + 1) * G] - t_ref) <= 1e-5 * np.maximum(1, np.abs(t_ref)))
            f_ref, _ = o.attention(g, np.arange(cfg.pages(b)), alpha)
            H.compare_out(full[b, g * G:(g + 1) * G], f_ref, cfg.dtype)


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25, 3.0])
def test_flat_scores_cluster_threshold(alpha):
    """Nearly equal keys put almost every token above every split's bound --
    more candidates than a split's slots hold -- so the threshold is solved by
    the whole cluster over every score.  129 pages per kv head (a ragged last
    page), every page listed; against the oracle on the same keys."""
    gen = torch.Generator().manual_seed(4242)
    H_kv, G, d, ps = 8, 4, 128, 64
    L = 128 * ps + 37
    P = (L + ps - 1) // ps
    sigma = 1e-4 if alpha == 2.0 else 0.02      # score spread small against the support's width
    keys = (sigma * torch.randn(H_kv, L, d, generator=gen)).to(torch.bfloat16)
    vals = torch.randn(H_kv, L, d, generator=gen).to(torch.bfloat16)
    q = torch.randn(1, H_kv * G, d, generator=gen)
    pool = B.Pool.allocate(P, H_kv, ps, d, torch.bfloat16, "cuda")
    pt = torch.arange(P, dtype=torch.int32, device="cuda").view(1, P)
    seq_lens = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = _status()
    B.append_metadata(pool, keys.cuda().unsqueeze(0).contiguous(), vals.cuda().unsqueeze(0).contiguous(), pt,
                      seq_lens, st)
    sel = torch.arange(P, dtype=torch.int32, device="cuda").view(1, 1, P).repeat(1, H_kv, 1).contiguous()
    cnt = torch.full((1, H_kv), P, dtype=torch.int32, device="cuda")
    ws = torch.empty(B.workspace_size(B.OP_SPARSE_ATTEND, 1, H_kv * G, H_kv, P, P, ps, d), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(1, H_kv * G, d, device="cuda")
    tau = torch.empty(1, H_kv * G, device="cuda")
    qd = q.cuda()
    scale = float(np.float32(1.0 / math.sqrt(d)))
    B.sparse_attend(pool, qd, pt, seq_lens, sel, cnt, alpha, scale, out, ws, st, tau_out=tau)
    _assert_ok(st)
    out, tau = out.cpu().numpy(), tau.cpu().numpy()
    qn = q[0].numpy()
    for g in range(0, H_kv, 3):
        K, V = keys[g].float().numpy(), vals[g].float().numpy()
        o_ref, t_ref, p = attend.entmax_attention(qn[g * G:(g + 1) * G], K, V, alpha, scale)
        # the case is the one meant: more candidates than the slots hold (16 x 256)
        # -- every token of the support is one; for alpha > 2 every token
        # within 1 of the largest score is one (the bound is max - 1 there)
        x = (alpha - 1.0) * scale * (K.astype(np.float64) @ qn[g * G:(g + 1) * G].astype(np.float64).T)
        for h in range(G):
            n_cand = np.count_nonzero(p[h]) if alpha <= 2.0 else np.count_nonzero(x[:, h] > x[:, h].max() - 1.0)
            assert n_cand > 16 * 256, n_cand
        H.compare_out(out[0, g * G:(g + 1) * G], o_ref, torch.bfloat16)
        assert np.all(np.abs(tau[0, g * G:(g + 1) * G] - t_ref) <= 1e-5 * np.maximum(1, np.abs(t_ref)))


def test_clustered_attention_longest_list():
    """The clustered kernel at its longest list: pages of 16 tokens, 4096
    listed pages per kv head (16 splits of 4096 tokens, the weighted-page
    bitmap full to its last word), a few planted tokens spread over the list
    (the first and the last page among them) carrying the support.  Output
    and tau against the oracle over every token, and the value pages loaded
    equal to the pages holding weight."""
    gen = torch.Generator().manual_seed(777)
    H_kv, G, d, ps, P = 2, 4, 128, 16, 4096
    L = P * ps
    keys = 0.1 * torch.randn(H_kv, L, d, generator=gen)
    vals = torch.randn(H_kv, L, d, generator=gen).to(torch.bfloat16)
    q = torch.randn(1, H_kv * G, d, generator=gen)
    plant = [3, 16 * 700 + 5, 16 * 2047 + 9, L - 2]          # tokens on pages 0, 700, 2047 and 4095
    for g in range(H_kv):
        for j, t in enumerate(plant):
            h = g * G + j % G
            keys[g, t] = 4.0 * q[0, h] / q[0, h].norm()
    keys = keys.to(torch.bfloat16)
    pool = B.Pool.allocate(P, H_kv, ps, d, torch.bfloat16, "cuda")
    pt = torch.arange(P, dtype=torch.int32, device="cuda").view(1, P)
    seq_lens = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = _status()
    B.append_metadata(pool, keys.cuda().unsqueeze(0).contiguous(), vals.cuda().unsqueeze(0).contiguous(), pt,
                      seq_lens, st)
    sel = torch.arange(P, dtype=torch.int32, device="cuda").view(1, 1, P).repeat(1, H_kv, 1).contiguous()
    cnt = torch.full((1, H_kv), P, dtype=torch.int32, device="cuda")
    ws = torch.empty(B.workspace_size(B.OP_SPARSE_ATTEND, 1, H_kv * G, H_kv, P, P, ps, d), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(1, H_kv * G, d, device="cuda")
    tau = torch.empty(1, H_kv * G, device="cuda")
    vp = torch.zeros(1, H_kv, dtype=torch.int32, device="cuda")
    scale = float(np.float32(1.0 / math.sqrt(d)))
    alpha = 1.5
    B.sparse_attend(pool, q.cuda(), pt, seq_lens, sel, cnt, alpha, scale, out, ws, st, tau_out=tau, v_pages=vp)
    _assert_ok(st)
    out, tau, vp = out.cpu().numpy(), tau.cpu().numpy(), vp.cpu().numpy()
    qn = q[0].numpy()
    for g in range(H_kv):
        K, V = keys[g].float().numpy(), vals[g].float().numpy()
        o_ref, t_ref, p = attend.entmax_attention(qn[g * G:(g + 1) * G], K, V, alpha, scale)
        H.compare_out(out[0, g * G:(g + 1) * G], o_ref, torch.bfloat16)
        assert np.all(np.abs(tau[0, g * G:(g + 1) * G] - t_ref) <= 1e-5 * np.maximum(1, np.abs(t_ref)))
        weighted = np.unique(np.nonzero(np.any(p > 0, axis=0))[0] // ps)
        assert 0 in weighted and P - 1 in weighted
        assert vp[0, g] == len(weighted), (vp[0, g], len(weighted))


def test_support_recovery_on_gpu():
    """If the kept pages hold the support, sparse == full (oracle: bitwise)."""
    wl = _wl(2, [8192 + 33])
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    o = H.OracleSeq(wl, 0)
    G = cfg.G
    sel = torch.zeros(1, cfg.H_kv, wl.max_pages, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, cfg.H_kv, dtype=torch.int32, device="cuda")
    for g in range(cfg.H_kv):
        _, _, pm = attend.entmax_attention(o.qgroup(g), o.keys[g], o.values[g], cfg.alpha, 1 / math.sqrt(cfg.d))
        sup_pages = set((np.nonzero(pm.sum(axis=0) > 0)[0] // cfg.ps).tolist())
        pages = sorted(sup_pages | {0, cfg.pages(0) - 1})
        sel[0, g, :len(pages)] = torch.tensor(pages, dtype=torch.int32)
        cnt[0, g] = len(pages)
    st = _status()
    ws = torch.empty(B.workspace_size(B.OP_SPARSE_ATTEND, 1, cfg.H_q, cfg.H_kv, wl.max_pages, wl.max_pages,
                                      cfg.ps, cfg.d), dtype=torch.uint8, device="cuda")
    out = torch.empty(1, cfg.H_q, cfg.d, device="cuda")
    B.sparse_attend(pool, wl.q, wl.page_table, seq_lens, sel, cnt, cfg.alpha, H.scale32(cfg), out, ws, st)
    wsf = torch.empty(B.workspace_size(B.OP_FULL_ENTMAX, 1, cfg.H_q, cfg.H_kv, wl.max_pages, 0, cfg.ps, cfg.d),
                      dtype=torch.uint8, device="cuda")
    full = torch.empty_like(out)
    B.full_entmax_decode(pool, wl.q, wl.page_table, seq_lens, cfg.alpha, H.scale32(cfg), full, wsf, st)
    _assert_ok(st)
    for g in range(cfg.H_kv):
        pages = sel[0, g, :cnt[0, g]].cpu().numpy()
        o_sp, _ = o.attention(g, pages, cfg.alpha)
        o_full, _ = o.attention(g, np.arange(cfg.pages(0)), cfg.alpha)
        assert np.array_equal(o_sp, o_full)            # oracle: exact
    assert torch.allclose(out, full, rtol=0, atol=H.BF16_ATOL)


def test_edge_cases_empty_sequence_and_full_budget():
    wl = _wl(2, [0, 64 * 5 + 1, 64])
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget=1000 if wl.max_pages >= 1000 else
                      wl.max_pages, alpha=cfg.alpha)
    step(wl.q)
    step.check()
    cnt = step.sel_count.cpu().numpy()
    assert np.all(cnt[0] == 0)
    assert np.all(cnt[1] == 6) and np.all(cnt[2] == 1)
    out, tau = step.out.cpu().numpy(), step.tau.cpu().numpy()
    assert np.all(out[0] == 0) and np.all(np.isinf(tau[0]))
    for b in (1, 2):
        o = H.OracleSeq(wl, b)
        for g in range(cfg.H_kv):
            o_ref, _ = o.attention(g, np.arange(cfg.pages(b)), cfg.alpha)
            H.compare_out(out[b, g * cfg.G:(g + 1) * cfg.G], o_ref, cfg.dtype)


def test_bad_page_id_reports_bounds():
    wl = _wl(2, [1000])
    pool, seq_lens = build_pool(wl)
    pt = wl.page_table.clone()
    pt[0, 3] = wl.num_phys + 11
    st = _status()
    ub = torch.empty(1, wl.cfg.H_kv, wl.max_pages, device="cuda")
    B.score_pages(pool, wl.q, pt, seq_lens, B.SCORE_BBOX, H.scale32(wl.cfg), st, ub=ub)
    torch.cuda.synchronize()
    assert int(st.item()) == B.DEVICE_BOUNDS


def test_host_validation_rejects_bad_arguments():
    wl = _wl(2, [100])
    pool, seq_lens = build_pool(wl)
    st = _status()
    out = torch.empty(1, wl.cfg.H_q, wl.cfg.d, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.EntmaxKVError) as e:
        B.full_entmax_decode(pool, wl.q, wl.page_table, seq_lens, 1.5, 0.1, out, small, st)
    assert e.value.code == B.WORKSPACE
    for alpha in (1.0, 0.5, 20.0):        # alpha-entmax needs alpha > 1; the library stops at 16
        with pytest.raises(B.EntmaxKVError) as e:
            B.full_entmax_decode(pool, wl.q, wl.page_table, seq_lens, alpha, 0.1, out, small, st)
        assert e.value.code == B.UNSUPPORTED


def test_bounded_wait_times_out_and_context_survives():
    st = _status()
    B.selftest_timeout(2_000_000, st)     # 2 ms
    torch.cuda.synchronize()
    assert int(st.item()) == B.TIMEOUT
    x = torch.arange(10, device="cuda").sum()
    assert int(x.item()) == 45


def test_decode_appends_then_step():
    """Config 5 shape: ragged batch, permuted pages, one token appended per step."""
    wl = _wl(5, [3000, 700, 64 * 9])
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 16, alpha=cfg.alpha)
    toks = []
    for t in range(3):
        k, v, q = wl.decode_token(t)
        step(q, k, v)
        toks.append((k, v, q))
    step.check()
    lens = [L + 3 for L in cfg.lengths]
    assert seq_lens.cpu().tolist() == lens
    out = step.out.cpu().numpy()
    q_last = toks[-1][2].cpu().numpy()
    G = cfg.G
    for b in range(cfg.B):
        keys, vals = H.host_sequence(wl, b)
        keys = np.concatenate([keys] + [t[0][b].float().cpu().numpy() for t in toks], axis=1)
        vals = np.concatenate([vals] + [t[1][b].float().cpu().numpy() for t in toks], axis=1)
        from oracle import replica
        for g in range(cfg.H_kv):
            meta = replica.page_meta(keys[g], cfg.ps)
            qg = q_last[b, g * G:(g + 1) * G]
            _, ubg = replica.bound(qg, meta["kmin"], meta["kmax"], H.scale32(cfg))
            P = (lens[b] + cfg.ps - 1) // cfg.ps
            pages = select.topk(ubg, select.budget_pages(P, -1, 1 / 16))
            tok = attend.token_indices(pages, lens[b], cfg.ps)
            o_ref, _, _ = attend.entmax_attention(qg, keys[g][tok], vals[g][tok], cfg.alpha, 1 / math.sqrt(cfg.d))
            H.compare_out(out[b, g * G:(g + 1) * G], o_ref, cfg.dtype)


def test_graphed_step_equals_eager_step():
    from sparse_long_context_min_b200.step import GraphedStep
    wl = _wl(2, [5000])
    cfg = wl.cfg
    pool_a, lens_a = build_pool(wl)
    pool_b, lens_b = build_pool(wl)
    eager = DecodeStep(pool_a, wl.page_table, lens_a, cfg.H_q, "topk", budget_frac=1 / 16, alpha=cfg.alpha)
    graphed = GraphedStep(DecodeStep(pool_b, wl.page_table, lens_b, cfg.H_q, "topk", budget_frac=1 / 16,
                                     alpha=cfg.alpha))
    for t in range(4):
        k, v, q = wl.decode_token(t)
        eager(q, k, v)
        if t % 2:   # one packed copy from pinned host memory
            graphed.inputs.copy_(graphed.pack_host(k, v, q), non_blocking=True)
        else:
            graphed.q.copy_(q)
            graphed.k.copy_(k)
            graphed.v.copy_(v)
        graphed.replay()
        torch.cuda.synchronize()
        assert torch.equal(eager.out, graphed.step.out)
        assert torch.equal(lens_a, lens_b)
    eager.check()
    graphed.step.check()
    # the same step writing its result straight into pinned host memory
    pool_c, lens_c = build_pool(wl)
    out_h = torch.empty(1, cfg.H_q, cfg.d, dtype=torch.float32).pin_memory()
    hosted = GraphedStep(DecodeStep(pool_c, wl.page_table, lens_c, cfg.H_q, "topk", budget_frac=1 / 16,
                                    alpha=cfg.alpha, out=out_h), stage_events=False)
    for t in range(4):
        k, v, q = wl.decode_token(t)
        hosted.inputs.copy_(hosted.pack_host(k, v, q), non_blocking=True)
        hosted.replay()
    torch.cuda.synchronize()
    hosted.step.check()
    assert torch.equal(out_h, graphed.step.out.cpu())
    stages = graphed.stage_us()
    assert set(stages) == set(GraphedStep.STAGES)
