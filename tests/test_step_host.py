"""Host orchestration of one decode step (step.DecodeStep) on the CPU.

The library calls are replaced by recorders, so this checks only what the
host side decides: the order of the calls, the buffers it allocates and
hands over (shapes and dtypes of the C ABI), and the page budget it sizes the
selection for.  The calls themselves run on the GPU in the gpu tests.
"""
import types

import pytest
import torch

from oracle import select
from sparse_long_context_min_b200 import binding as B
from sparse_long_context_min_b200 import step as S


@pytest.fixture
def calls(monkeypatch):
    log = []

    def rec(name):
        def f(*args, **kw):
            log.append((name, args, kw))
        return f

    for name in ("append_metadata", "append_score_pages", "score_pages", "select", "sparse_attend"):
        monkeypatch.setattr(B, name, rec(name))
    monkeypatch.setattr(B, "workspace_size", lambda *a: 4096)
    return log


def _pool(H_kv=8, ps=64, d=128):
    return types.SimpleNamespace(H_kv=H_kv, ps=ps, d=d, k_pool=torch.empty(0, dtype=torch.bfloat16))


@pytest.mark.parametrize("frac", [1 / 64, 1 / 16, 1 / 8])
def test_topk_step_calls_and_buffers(calls, frac):
    Bn, H_q, max_pages = 2, 32, 1000
    pt = torch.zeros(Bn, max_pages, dtype=torch.int32)
    lens = torch.tensor([64 * 999, 5], dtype=torch.int32)
    st = S.DecodeStep(_pool(), pt, lens, H_q, "topk", budget_frac=frac)
    # room for the largest selection the library can make: ceil(f * P_b) <= ceil(f * max_pages)
    assert st.k_max == select.budget_pages(max_pages, -1, frac)
    q = torch.zeros(Bn, H_q, 128)
    k = torch.zeros(Bn, 8, 1, 128, dtype=torch.bfloat16)
    st(q, k, k)
    # top-k: the token append and the bounding-box scoring are one library call
    assert [c[0] for c in calls] == ["append_score_pages", "select", "sparse_attend"]
    _, as_args, _ = calls[0]
    assert as_args[1] is k and as_args[3] is q and tuple(as_args[8].shape) == (Bn, 8, max_pages)
    calls.clear()
    st(q)                                            # no token: scoring alone
    assert [c[0] for c in calls] == ["score_pages", "select", "sparse_attend"]
    _, score_args, score_kw = calls[0]
    assert score_args[4] == B.SCORE_BBOX and tuple(score_kw["ub"].shape) == (Bn, 8, max_pages)
    _, sel_args, sel_kw = calls[1]
    assert sel_args[0] == B.SELECT_TOPK and sel_kw["budget_frac"] == frac and sel_kw["budget"] == -1
    assert tuple(st.sel.shape) == (Bn, 8, st.k_max) and st.sel.dtype == torch.int32
    assert tuple(st.sel_count.shape) == (Bn, 8) and st.sel_count.dtype == torch.int32
    assert tuple(st.out.shape) == (Bn, H_q, 128) and st.out.dtype == torch.float32
    assert tuple(st.tau.shape) == (Bn, H_q) and st.workspace.numel() >= 4096
    _, att_args, att_kw = calls[2]
    assert att_args[4] is st.sel and att_args[5] is st.sel_count and att_kw["tau_out"] is st.tau


def test_gauss_step_sizes_for_every_page(calls):
    Bn, H_q, max_pages = 1, 32, 300
    st = S.DecodeStep(_pool(), torch.zeros(Bn, max_pages, dtype=torch.int32), torch.tensor([64 * 300]), H_q,
                      "gauss", alpha=2.0, delta=0.5)
    assert st.k_max == max_pages
    st(torch.zeros(Bn, H_q, 128))
    assert [c[0] for c in calls] == ["score_pages", "select", "sparse_attend"]   # no token to append
    _, score_args, score_kw = calls[0]
    assert score_args[4] == B.SCORE_GAUSS
    assert all(tuple(score_kw[k].shape) == (Bn, H_q, max_pages) for k in ("m", "v", "est_max"))
    _, sel_args, sel_kw = calls[1]
    assert sel_args[0] == B.SELECT_GAUSS and sel_kw["alpha"] == 2.0 and sel_kw["delta"] == 0.5
    assert tuple(sel_kw["tau_hat"].shape) == (Bn, H_q)


def test_fixed_budget_and_caller_output(calls):
    out = torch.empty(1, 32, 128)
    st = S.DecodeStep(_pool(), torch.zeros(1, 50, dtype=torch.int32), torch.tensor([64 * 50]), 32, "topk",
                      budget=7, out=out)
    assert st.k_max == 7 and st.out is out
    st.attend(torch.zeros(1, 32, 128))
    assert calls[-1][1][8] is out


def test_gauss_step_appends_then_scores(calls):
    st = S.DecodeStep(_pool(), torch.zeros(1, 30, dtype=torch.int32), torch.tensor([64 * 20]), 32, "gauss")
    k = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16)
    st(torch.zeros(1, 32, 128), k, k)
    assert [c[0] for c in calls] == ["append_metadata", "score_pages", "select", "sparse_attend"]
