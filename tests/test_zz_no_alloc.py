"""entmaxkv_sparse_attend_static: sparse attention without a caller workspace.

Some callers cannot allocate device memory while they decode (code under CUDA
stream capture, hosts whose allocator owns all device memory, loops where an
allocation would synchronise the device).  The static entry point takes its
scratch from a buffer built into the library.  This file is collected last on
purpose: a failure here leaves every other test already run.  It checks, on
two calls in a row, that the static entry point gives the same output as the
workspace entry point within the attention tolerance, and that a problem too
large for the buffer is refused.
"""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

from sparse_long_context_min_b200 import binding as B
from sparse_long_context_min_b200 import workloads
from sparse_long_context_min_b200.step import DecodeStep, build_pool

pytestmark = pytest.mark.gpu

BF16_ATOL = 2e-3   # the bf16-cache attention tolerance used by the parity tests


def test_static_scratch_matches_workspace_entry_point_twice():
    cfg = replace(workloads.config(2), lengths=[20000])
    wl = workloads.Workload(cfg, device="cuda")
    pool, seq_lens = build_pool(wl)
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 16, alpha=cfg.alpha)
    scale = float(np.float32(1.0 / math.sqrt(cfg.d)))
    for call in range(2):
        k, v, q = wl.decode_token(call)
        step(q, k, v)                       # append, score, select, attend (workspace path)
        step.check()
        ref = step.out.clone()
        ref_tau = step.tau.clone()
        out = torch.full_like(ref, float("nan"))
        tau = torch.full_like(ref_tau, float("nan"))
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        B.sparse_attend_static(pool, q, wl.page_table, seq_lens, step.sel, step.sel_count, cfg.alpha, scale,
                               out, st, tau_out=tau)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, B.status_string(int(st.item()))
        assert torch.isfinite(out).all()
        assert (out - ref).abs().max().item() <= BF16_ATOL
        assert (tau - ref_tau).abs().max().item() <= 1e-5 * max(1.0, ref_tau.abs().max().item())


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
