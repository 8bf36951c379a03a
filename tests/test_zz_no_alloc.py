"""entmaxkv_sparse_attend_static: sparse attention without a caller workspace.

Some callers cannot allocate device memory while they decode: code under CUDA
stream capture (allocation is not allowed while capturing), hosts whose own
allocator owns all device memory, and loops where an allocation would
synchronise the device.  The static entry point takes its scratch from a
buffer built into the library.  This file is collected last on purpose: a
failure here leaves every other test already run.

It checks, on consecutive calls, that the static entry point gives exactly the
workspace entry point's output (the same kernels with the same split count and
a fixed-order split reduction, so bit for bit) and the oracle's within the
attention tolerance, also after a larger call has left other data at the
offsets a smaller call reuses; and that a problem too large for the buffer is
refused.
"""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import attend
from sparse_long_context_min_b200 import binding as B
from sparse_long_context_min_b200 import workloads
from sparse_long_context_min_b200.step import DecodeStep, build_pool

pytestmark = pytest.mark.gpu

BF16_ATOL = 2e-3   # the bf16-cache attention tolerance used by the parity tests


def _static(step, pool, wl, q, alpha, scale):
    out = torch.full_like(step.out, float("nan"))
    tau = torch.full_like(step.tau, float("nan"))
    vp = torch.zeros_like(step.v_pages)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.sparse_attend_static(pool, q, wl.page_table, step.seq_lens, step.sel, step.sel_count, alpha, scale,
                           out, st, tau_out=tau, v_pages=vp)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, B.status_string(int(st.item()))
    return out, tau, vp


def _oracle_out(wl, toks, b, g, pages, alpha):
    cfg = wl.cfg
    keys, vals = wl.sequence(b, heads=[g])
    keys, vals = keys[0].float().cpu().numpy(), vals[0].float().cpu().numpy()
    if toks:
        keys = np.concatenate([keys] + [t[0][b, g].float().cpu().numpy() for t in toks], axis=0)
        vals = np.concatenate([vals] + [t[1][b, g].float().cpu().numpy() for t in toks], axis=0)
    q = toks[-1][2][b].cpu().numpy() if toks else wl.q[b].cpu().numpy()
    tok = attend.token_indices(pages, keys.shape[0], cfg.ps)
    G = cfg.G
    o, _, _ = attend.entmax_attention(q[g * G:(g + 1) * G], keys[tok], vals[tok], alpha, 1 / math.sqrt(cfg.d))
    return o


def test_static_scratch_matches_workspace_entry_point_and_oracle():
    # a larger problem first (4 sequences, a bigger budget): its scores, partial
    # outputs and counters are left in the buffer where the smaller calls' land
    big = workloads.Workload(replace(workloads.config(2), B=4, lengths=[30000, 20000, 25000, 9000]), device="cuda")
    bpool, blens = build_pool(big)
    bstep = DecodeStep(bpool, big.page_table, blens, big.cfg.H_q, "topk", budget_frac=1 / 4, alpha=big.cfg.alpha)
    bstep(big.q)
    bstep.check()
    scale = float(np.float32(1.0 / math.sqrt(big.cfg.d)))
    bout, _, _ = _static(bstep, bpool, big, big.q, big.cfg.alpha, scale)
    assert torch.equal(bout, bstep.out)

    cfg = replace(workloads.config(2), lengths=[20000])
    wl = workloads.Workload(cfg, device="cuda")
    pool, seq_lens = build_pool(wl)
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 16, alpha=cfg.alpha)
    toks = []
    for call in range(2):
        k, v, q = wl.decode_token(call)
        toks.append((k, v, q))
        step.v_pages.zero_()
        step(q, k, v)                       # append, score, select, attend (workspace path)
        step.check()
        out, tau, vp = _static(step, pool, wl, q, cfg.alpha, scale)
        assert torch.equal(out, step.out)
        assert torch.equal(tau, step.tau)
        assert torch.equal(vp, step.v_pages)
        sel, cnt, o = step.sel.cpu().numpy(), step.sel_count.cpu().numpy(), out.cpu().numpy()
        G = cfg.G
        for g in (0, 5):
            o_ref = _oracle_out(wl, toks, 0, g, sel[0, g, :cnt[0, g]], cfg.alpha)
            assert np.abs(o[0, g * G:(g + 1) * G] - o_ref).max() <= BF16_ATOL


def test_static_scratch_refuses_problems_beyond_the_buffer():
    pool = B.Pool.allocate(16, 8, 64, 128)
    q = torch.zeros(64, 32, 128, device="cuda")
    pt = torch.zeros(64, 20000, dtype=torch.int32, device="cuda")
    lens = torch.zeros(64, dtype=torch.int32, device="cuda")
    sel = torch.zeros(64, 8, 20000, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(64, 8, dtype=torch.int32, device="cuda")
    out = torch.empty(64, 32, 128, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    need = B.workspace_size(B.OP_SPARSE_ATTEND, 64, 32, 8, 20000, 20000, 64, 128)
    assert need > B.STATIC_SCRATCH_BYTES
    with pytest.raises(B.EntmaxKVError) as e:
        B.sparse_attend_static(pool, q, pt, lens, sel, cnt, 1.5, 0.088, out, st)
    assert e.value.code == B.STATIC_LIMIT
    assert "built-in buffer" in B.status_string(B.STATIC_LIMIT)
