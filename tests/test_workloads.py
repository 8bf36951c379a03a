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
