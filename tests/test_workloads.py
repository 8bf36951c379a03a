"""Host-side checks of the seeded workload generator (no GPU)."""
import torch

from sparse_long_context_min_b200 import workloads


def test_configs_match_the_benchmark_suite():
    c1, c2, c3, c4 = (workloads.config(n) for n in (1, 2, 3, 4))
    assert (c1.B, c1.H_q, c1.H_kv, c1.d, c1.lengths, c1.ps, c1.dtype) == (1, 4, 1, 64, [4096], 16, torch.float32)
    assert c1.pages(0) == 256 and c1.budgets == [32]
    assert (c2.H_q, c2.H_kv, c2.d, c2.ps, c2.lengths) == (32, 8, 128, 64, [131072])
    assert [b * 2048 for b in (1 / 32, 1 / 16, 1 / 8)] == c2.budgets
    assert c3.B == 4 and c3.centres == "walk" and c3.alphas == [1.5, 2.0] and c3.deltas == [0.0, 0.5, 1.0]
    assert c4.lengths == [1 << 20] and c4.pages(0) == 16384 and c4.budget_frac == 1 / 64
    c5 = workloads.config(5, B=32)
    assert c5.B == 32 and all(32768 <= L <= 524288 for L in c5.lengths) and c5.permute_pages


def test_generation_is_deterministic_and_shaped():
    cfg = workloads.config(2, L=1000)
    a = workloads.Workload(cfg)
    b = workloads.Workload(cfg)
    assert torch.equal(a.q, b.q)
    ka, va = a.sequence(0)
    kb, vb = b.sequence(0)
    assert torch.equal(ka, kb) and torch.equal(va, vb)
    assert ka.shape == (8, 1000, 128) and ka.dtype == torch.bfloat16
    planted = a.planted(0)
    assert sum(len(v) for v in planted.values()) == 64 * 8      # 64 per kv head
    # a planted key points along its query head
    h, pos = next((h, p) for h, p in planted.items() if p)
    qh = a.q[0, h] / a.q[0, h].norm()
    cos = (ka[h // 4, pos[0]].float() @ qh) / ka[h // 4, pos[0]].float().norm()
    assert cos > 0.9


def test_permuted_page_tables_are_a_partition():
    cfg = workloads.config(5, B=4)
    cfg.lengths[:] = [100, 2000, 64, 640]
    wl = workloads.Workload(cfg)
    used = []
    for b in range(cfg.B):
        used += wl.page_table[b, :cfg.pages(b) + wl.extra_pages].tolist()
    assert sorted(used) == list(range(wl.num_phys))


def test_walk_centres_and_short_sequences():
    import dataclasses
    cfg = dataclasses.replace(workloads.config(3), B=2, lengths=[0, 300])
    wl = workloads.Workload(cfg)
    k0, _ = wl.sequence(0)
    k1, _ = wl.sequence(1)
    assert k0.shape == (8, 0, 128) and k1.shape == (8, 300, 128)


def _page_stats(keys, ps, planted_pos):
    """Page means and within-page deviations of one kv head's keys, planted tokens left out."""
    k = keys.float()
    L = k.shape[0]
    P = L // ps
    mask = torch.ones(L, dtype=torch.bool)
    mask[list(planted_pos)] = False
    means, dev = [], []
    for p in range(P):
        blk = k[p * ps:(p + 1) * ps][mask[p * ps:(p + 1) * ps]]
        mu = blk.mean(0)
        means.append(mu)
        dev.append(blk - mu)
    return torch.stack(means), torch.cat(dev)


def test_clustered_keys_follow_the_recipe():
    """Centres N(0, I) per (page, kv head), tokens centre + 0.3 N(0, I)."""
    import dataclasses
    cfg = dataclasses.replace(workloads.config(2), lengths=[64 * 200])
    wl = workloads.Workload(cfg)
    keys, vals = wl.sequence(0, heads=[0])
    planted = [p for h in range(cfg.G) for p in wl.planted(0).get(h, [])]
    means, dev = _page_stats(keys[0], cfg.ps, planted)
    assert 0.93 < float(means.std()) < 1.07
    assert 0.29 < float(dev.std()) < 0.31
    assert abs(float(vals.float().mean())) < 0.01 and 0.98 < float(vals.float().std()) < 1.02
    assert 0.97 < float(wl.q.std()) < 1.03


def test_walk_centres_follow_the_recipe():
    """c_{p+1} = 0.9 c_p + 0.44 N(0, I): lag-one correlation 0.9 and variance
    near the stationary 0.44^2 / (1 - 0.81) = 1.02; tokens spread 0.5."""
    import dataclasses
    cfg = dataclasses.replace(workloads.config(3), B=1, lengths=[64 * 600])
    wl = workloads.Workload(cfg)
    keys, _ = wl.sequence(0, heads=[2])
    planted = [p for h in range(2 * cfg.G, 3 * cfg.G) for p in wl.planted(0).get(h, [])]
    means, dev = _page_stats(keys[0], cfg.ps, planted)
    a, b = means[:-1], means[1:]
    corr = float(((a - a.mean(0)) * (b - b.mean(0))).mean() / (a.std() * b.std()))
    assert 0.85 < corr < 0.94
    assert 0.8 < float(means.var()) < 1.25
    assert 0.48 < float(dev.std()) < 0.52
    counts = [len(v) for v in wl.planted(0).values()]
    assert len(counts) == cfg.H_q and all(16 <= c <= 512 for c in counts)
