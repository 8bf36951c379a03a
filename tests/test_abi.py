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
    rc = lib.entmaxkv_select(B.SELECT_GAUSS, None, None, None, None, None, 64, 1, 32, 8, 100, -1, 0.0, 1.02,
                             0.5, 100, None, None, None, None, 0, st, None)
    assert rc == B.UNSUPPORTED           # the Gaussian selector's quadrature covers alpha >= 1.05
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


def test_static_entry_checks_arguments_before_its_size():
    """entmaxkv_sparse_attend_static runs entmaxkv_sparse_attend's argument
    checks before comparing the problem with its built-in buffer, so a bad
    call gets the same code from both entry points; a valid oversized call is
    refused with ENTMAXKV_STATIC_LIMIT.  Nothing here reaches the GPU."""
    lib = B.lib()
    st = ctypes.c_void_p(16)
    pool = B.CPool(16, 16, 16, 16, 16, 16, 16, 10, 8, 64, 128, B.BF16)
    Bn, H_q, max_pages, k_max = 64, 32, 20000, 20000       # far beyond the buffer
    assert B.workspace_size(B.OP_SPARSE_ATTEND, Bn, H_q, 8, max_pages, k_max, 64, 128) > B.STATIC_SCRATCH_BYTES

    def call(alpha=1.5, scale=0.088, H=H_q, sel=ctypes.c_void_p(16), out=ctypes.c_void_p(16)):
        return lib.entmaxkv_sparse_attend_static(ctypes.byref(pool), ctypes.c_void_p(16), H, ctypes.c_void_p(16),
                                                 max_pages, ctypes.c_void_p(16), Bn, sel, ctypes.c_void_p(16),
                                                 k_max, ctypes.c_float(alpha), ctypes.c_float(scale), out, None,
                                                 None, st, None)

    assert call(alpha=1.0) == B.UNSUPPORTED                 # alpha-entmax needs alpha > 1
    assert call(alpha=20.0) == B.UNSUPPORTED
    assert call(scale=-1.0) == B.INVALID_ARG
    assert call(H=30) == B.INVALID_ARG                       # 30 query heads over 8 kv heads
    assert call(H=24) == B.UNSUPPORTED                       # group of 3
    assert call(sel=None) == B.INVALID_ARG                   # no page list
    assert call(out=None) == B.INVALID_ARG
    assert call() == B.STATIC_LIMIT
