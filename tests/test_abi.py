"""The C-ABI library loads and exports every entry point include/entmaxkv.h declares.

Host-only entry points (status strings, workspace sizes, argument validation that
fails before any launch) are exercised without a GPU.
"""
import ctypes
import os
import re

import pytest

from sparse_long_context_min_b200 import binding as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "entmaxkv.h")


def declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ENTMAXKV_API\s+[\w\s\*]+?\b(entmaxkv_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared()
    assert len(names) >= 9
    lib = B.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.SYMBOLS)


def test_status_strings():
    assert B.status_string(0) == "ok"
    assert "timed out" in B.status_string(B.TIMEOUT)
    assert B.status_string(99) == "unknown status"


def test_workspace_sizes():
    big = B.workspace_size(B.OP_FULL_ENTMAX, 1, 32, 8, 16385, 0, 64, 128)
    small = B.workspace_size(B.OP_SPARSE_ATTEND, 1, 32, 8, 16385, 256, 64, 128)
    assert big >= 1 * 32 * 16385 * 64 * 4          # one score per listed token and head
    assert 32 * 256 * 64 * 4 <= small < big
    assert B.workspace_size(B.OP_FULL_SOFTMAX, 1, 32, 8, 16385, 0, 64, 128) < small
    assert B.workspace_size(B.OP_SELECT, 1, 32, 8, 16385, 256, 64, 128) == 0
    assert B.workspace_size(B.OP_SPARSE_ATTEND, 0, 32, 8, 10, 1, 64, 128) == 0
    # sparse softmax keeps no scores: partials and merge terms only
    sm = B.workspace_size(B.OP_SPARSE_SOFTMAX, 1, 32, 8, 16385, 256, 64, 128)
    assert 0 < sm < small
    assert B.workspace_size(B.OP_SPARSE_SOFTMAX, 1, 32, 8, 16385, 0, 64, 128) == 0


def test_host_validation_without_gpu():
    lib = B.lib()
    st = ctypes.c_void_p(16)       # never dereferenced: validation fails first
    pool = B.CPool(16, 16, 16, 16, 16, 16, 16, 10, 8, 64, 96, B.BF16)   # d = 96 unsupported
    rc = lib.entmaxkv_score_pages(ctypes.byref(pool), ctypes.c_void_p(16), 32, ctypes.c_void_p(16), 10,
                                  ctypes.c_void_p(16), 1, B.SCORE_BBOX, 0.1, ctypes.c_void_p(16), None,
                                  None, None, st, None)
    assert rc == B.UNSUPPORTED
    pool = B.CPool(16, 16, 16, 16, 16, 16, 16, 10, 8, 64, 128, B.BF16)
    rc = lib.entmaxkv_score_pages(ctypes.byref(pool), ctypes.c_void_p(16), 30, ctypes.c_void_p(16), 10,
                                  ctypes.c_void_p(16), 1, B.SCORE_BBOX, 0.1, ctypes.c_void_p(16), None,
                                  None, None, st, None)
    assert rc == B.INVALID_ARG           # 30 query heads over 8 kv heads
    rc = lib.entmaxkv_selftest_timeout(-1, st, None)
    assert rc == B.INVALID_ARG
    rc = lib.entmaxkv_select(B.SELECT_TOPK, None, None, None, None, None, 64, 1, 32, 8, 100, 300, 0.0, 1.5,
                             0.0, 256, None, None, None, None, 0, st, None)
    assert rc == B.INVALID_ARG           # budget above k_max
    pool = B.CPool(16, 16, 16, 16, 16, 16, 16, 10, 8, 64, 128, B.BF16)
    rc = lib.entmaxkv_sparse_softmax_attend(ctypes.byref(pool), ctypes.c_void_p(16), 32, ctypes.c_void_p(16), 10,
                                            ctypes.c_void_p(16), 1, None, None, 4, 0.1, ctypes.c_void_p(16),
                                            ctypes.c_void_p(256), 1 << 20, st, None)
    assert rc == B.INVALID_ARG           # no page list
    rc = lib.entmaxkv_select(B.SELECT_GAUSS, None, None, None, None, None, 64, 1, 32, 8, 100, -1, 0.0, 1.1,
                             0.5, 100, None, None, None, None, 0, st, None)
    assert rc == B.UNSUPPORTED           # the Gaussian selector's quadrature covers alpha >= 1.25
    rc = lib.entmaxkv_full_entmax_decode(ctypes.byref(pool), ctypes.c_void_p(16), 32, ctypes.c_void_p(16), 10,
                                         ctypes.c_void_p(16), 1, 1.0, 0.1, ctypes.c_void_p(16), None, None,
                                         ctypes.c_void_p(256), 1 << 20, st, None)
    assert rc == B.UNSUPPORTED           # alpha must exceed 1


@pytest.mark.parametrize("B_", [0])
def test_empty_batch_is_a_noop(B_):
    lib = B.lib()
    pool = B.CPool(16, 16, 16, 16, 16, 16, 16, 10, 8, 64, 128, B.BF16)
    rc = lib.entmaxkv_append_metadata(ctypes.byref(pool), None, None, 1, None, 10, None, B_, None, None)
    assert rc == B.OK
