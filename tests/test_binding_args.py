"""The Python binding refuses tensors the C ABI cannot check, before any call.

The library takes plain pointers and sizes, so a tensor of the wrong dtype, a
strided view, a buffer smaller than the sizes passed, or pageable host memory
would be read or written out of bounds (or at an address the GPU cannot
reach).  The binding checks each tensor first; these tests run on the CPU with
the library replaced by a stub that fails if it is ever reached.
"""
import types

import pytest
import torch

from sparse_long_context_min_b200 import binding as B


@pytest.fixture(autouse=True)
def no_library(monkeypatch):
    def unreachable():
        raise AssertionError("the library was called although an argument was invalid")
    monkeypatch.setattr(B, "lib", unreachable)


def _pool(H_kv=8, d=128, dtype=torch.bfloat16):
    # what the entry points read from a Pool before the library call
    return types.SimpleNamespace(H_kv=H_kv, d=d, k_pool=torch.empty(0, dtype=dtype))


def _i32(*shape):
    return torch.zeros(*shape, dtype=torch.int32)


def _f32(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


def _raises(fn, *words):
    with pytest.raises(B.EntmaxKVError) as e:
        fn()
    assert e.value.code == B.INVALID_ARG
    for w in words:
        assert w in str(e.value), str(e.value)


def _score(**over):
    a = dict(q=_f32(2, 32, 128), page_table=_i32(2, 10), seq_lens=_i32(2), status=_i32(1), ub=_f32(2, 8, 10))
    a.update(over)
    return lambda: B.score_pages(_pool(), a["q"], a["page_table"], a["seq_lens"], B.SCORE_BBOX, 0.1,
                                 a["status"], ub=a["ub"])


def test_score_pages_arguments():
    _raises(_score(q=torch.zeros(2, 32, 128, dtype=torch.float64)), "q must be torch.float32")
    _raises(_score(q=_f32(2, 128, 32).transpose(1, 2)), "q must be contiguous")
    _raises(_score(q=_f32(2, 32, 64)), "64 dims per head")
    _raises(_score(q=_f32(2, 32 * 128)), "q must have 3 dimensions")
    _raises(_score(page_table=torch.zeros(2, 10, dtype=torch.int64)), "page_table must be torch.int32")
    _raises(_score(page_table=_i32(1, 10)), "1 rows for 2 sequences")
    _raises(_score(seq_lens=_i32(1)), "seq_lens holds 1 elements; the call addresses 2")
    _raises(_score(ub=_f32(2, 8, 9)), "ub holds 144 elements; the call addresses 160")
    _raises(_score(ub=None), "ub is required")
    _raises(_score(status=_i32(0)), "status holds 0")
    # every tensor well-formed, but in pageable host memory
    _raises(_score(), "must be in device memory or pinned host memory")


def test_gauss_scoring_needs_query_head_sized_outputs():
    m = _f32(2, 32, 10)
    fn = lambda v: lambda: B.score_pages(_pool(), _f32(2, 32, 128), _i32(2, 10), _i32(2), B.SCORE_GAUSS, 0.1,
                                         _i32(1), m=m, v=v, est_max=m)
    _raises(fn(_f32(2, 8, 10)), "v holds 160 elements; the call addresses 640")
    _raises(fn(None), "v is required")


def test_append_arguments():
    pool = _pool()
    k = torch.zeros(2, 8, 3, 128, dtype=torch.bfloat16)
    call = lambda k_, v_: lambda: B.append_metadata(pool, k_, v_, _i32(2, 10), _i32(2), _i32(1))
    _raises(call(k.float(), k), "k_new must be torch.bfloat16")
    _raises(call(torch.zeros(2, 4, 3, 128, dtype=torch.bfloat16), k), "k_new must be [B, 8, n_new, 128]")
    _raises(call(k, torch.zeros(2, 8, 2, 128, dtype=torch.bfloat16)), "v_new holds")
    _raises(call(k, k), "pinned host memory")


def test_select_arguments():
    sl = _i32(2)
    topk = lambda sel, cnt, ub: lambda: B.select(B.SELECT_TOPK, sl, 64, 32, 8, 100, 16, sel, cnt, _i32(1), ub=ub,
                                                 budget=16)
    _raises(topk(_i32(2, 8, 15), _i32(2, 8), _f32(2, 8, 100)), "sel holds 240 elements; the call addresses 256")
    _raises(topk(_i32(2, 8, 16), _i32(2, 7), _f32(2, 8, 100)), "sel_count holds 14")
    _raises(topk(_i32(2, 8, 16), _i32(2, 8), _f32(2, 8, 99)), "ub holds")
    _raises(lambda: B.select(B.SELECT_TOPK, _i32(2, 1), 64, 32, 8, 100, 16, _i32(2, 8, 16), _i32(2, 8), _i32(1),
                             ub=_f32(2, 8, 100)), "seq_lens must have 1 dimensions")
    m = _f32(2, 32, 100)
    _raises(lambda: B.select(B.SELECT_GAUSS, sl, 64, 32, 8, 100, 100, _i32(2, 8, 100), _i32(2, 8), _i32(1),
                             m=m, v=m, est_max=m, alpha=1.5, delta=0.5), "tau_hat is required")


def _attend(**over):
    a = dict(q=_f32(2, 32, 128), page_table=_i32(2, 10), seq_lens=_i32(2), sel=_i32(2, 8, 4), cnt=_i32(2, 8),
             out=_f32(2, 32, 128), ws=torch.zeros(64, dtype=torch.uint8), status=_i32(1), tau=None, vp=None)
    a.update(over)
    return lambda: B.sparse_attend(_pool(), a["q"], a["page_table"], a["seq_lens"], a["sel"], a["cnt"], 1.5, 0.1,
                                   a["out"], a["ws"], a["status"], tau_out=a["tau"], v_pages=a["vp"])


def test_attention_arguments():
    _raises(_attend(sel=_i32(2, 4, 8)), "sel must be [B, H_kv, k_max] with B = 2 and H_kv = 8")
    _raises(_attend(sel=_i32(1, 8, 4)), "sel must be [B, H_kv, k_max]")
    _raises(_attend(sel=_i32(2, 8, 4).long()), "sel must be torch.int32")
    _raises(_attend(out=_f32(2, 32, 127)), "out holds")
    _raises(_attend(tau=_f32(2, 31)), "tau_out holds 62 elements; the call addresses 64")
    _raises(_attend(vp=_f32(2, 8)), "v_pages must be torch.int32")
    _raises(_attend(ws=torch.zeros(64, 2, dtype=torch.uint8)[:, 0]), "workspace must be contiguous")
    _raises(_attend(), "pinned host memory")
    # the other attention entry points share the checks
    _raises(lambda: B.full_softmax_decode(_pool(), _f32(2, 32, 128), _i32(2, 10), _i32(2), 0.1, _f32(2, 32, 64),
                                          torch.zeros(64, dtype=torch.uint8), _i32(1)), "out holds")
    _raises(lambda: B.sparse_softmax_attend(_pool(), _f32(2, 32, 128), _i32(2, 10), _i32(2), _i32(2, 8, 4),
                                            _i32(2, 3), 0.1, _f32(2, 32, 128), torch.zeros(64, dtype=torch.uint8),
                                            _i32(1)), "sel_count holds 6")
    _raises(lambda: B.sparse_attend_static(_pool(), _f32(2, 32, 128), _i32(2, 10), _i32(2), _i32(2, 8, 4),
                                           _i32(2, 8), 1.5, 0.1, _f32(2, 32, 128), _i32(1), tau_out=_f32(1)),
            "tau_out holds 1")
    _raises(lambda: B.full_entmax_decode(_pool(), _f32(2, 32, 128), _i32(2, 10), _i32(2), 1.5, 0.1,
                                         _f32(2, 32, 128), None, _i32(1)), "workspace is required")
    _raises(lambda: B.selftest_timeout(1000, _f32(1)), "status must be torch.int32")


def test_pool_arguments():
    kv = torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16)
    meta = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    f = torch.zeros(4, 2, 64)
    with pytest.raises(B.EntmaxKVError) as e:
        B.Pool(kv.half(), kv.half(), meta, meta, f, f, _i32(4))
    assert e.value.code == B.UNSUPPORTED
    _raises(lambda: B.Pool(kv, kv[:3], meta, meta, f, f, _i32(4)), "v_pool holds")
    _raises(lambda: B.Pool(kv, kv, meta.float(), meta, f, f, _i32(4)), "kmin must be torch.bfloat16")
    _raises(lambda: B.Pool(kv, kv, meta, meta, f, f[:3], _i32(4)), "m2 holds")
    _raises(lambda: B.Pool(kv, kv, meta, meta, f, f, _i32(3)), "count holds 3")
    _raises(lambda: B.Pool(kv, kv, meta, meta, f, f, _i32(4)), "pinned host memory")
