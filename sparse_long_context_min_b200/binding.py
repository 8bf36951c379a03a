"""Thin ctypes binding over the EntmaxKV C ABI (include/entmaxkv.h).

Argument marshalling only: every function below checks that each tensor can
be handed to the library as a plain pointer (dtype, dense layout, enough
elements for the sizes the call passes, memory the current GPU can address),
then passes the tensors' pointers, sizes and the current CUDA stream to the
entry point of the same name and raises on a non-zero host status.  All work
runs in the CUDA library; there is no other implementation to fall back to --
if the shared library is missing the first call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libentmaxkv.so")

OK, INVALID_ARG, UNSUPPORTED, CUDA_ERROR, TIMEOUT, DEVICE_BOUNDS, WORKSPACE, STATIC_LIMIT = range(8)
STATIC_SCRATCH_BYTES = 16 << 20
F32, BF16 = 0, 1
SCORE_BBOX, SCORE_GAUSS = 0, 1
SELECT_TOPK, SELECT_GAUSS = 0, 1
OP_SELECT, OP_SPARSE_ATTEND, OP_FULL_ENTMAX, OP_FULL_SOFTMAX, OP_SPARSE_SOFTMAX = range(5)

# every symbol the header declares (checked by the tests)
SYMBOLS = (
    "entmaxkv_append_metadata", "entmaxkv_score_pages", "entmaxkv_select", "entmaxkv_sparse_attend",
    "entmaxkv_full_entmax_decode", "entmaxkv_full_softmax_decode", "entmaxkv_workspace_size",
    "entmaxkv_status_string", "entmaxkv_selftest_timeout", "entmaxkv_sparse_attend_static",
    "entmaxkv_sparse_softmax_attend", "entmaxkv_append_score_pages",
)


class EntmaxKVError(RuntimeError):
    def __init__(self, code, where, detail=None):
        super().__init__("%s: %s (status %d)" % (where, detail or status_string(code), code))
        self.code = code


class CPool(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("kmin", ctypes.c_void_p), ("kmax", ctypes.c_void_p),
                ("mean", ctypes.c_void_p), ("m2", ctypes.c_void_p), ("count", ctypes.c_void_p),
                ("num_phys_pages", ctypes.c_int32), ("H_kv", ctypes.c_int32), ("ps", ctypes.c_int32),
                ("d", ctypes.c_int32), ("dtype", ctypes.c_int32)]


_lib = None


def lib():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("EntmaxKV CUDA library not built (%s missing); run "
                               "`python -m sparse_long_context_min_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, I, F, S = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
        PP = ctypes.POINTER(CPool)
        L.entmaxkv_append_metadata.argtypes = [PP, P, P, I, P, I, P, I, P, P]
        L.entmaxkv_score_pages.argtypes = [PP, P, I, P, I, P, I, I, F, P, P, P, P, P, P]
        L.entmaxkv_select.argtypes = [I, P, P, P, P, P, I, I, I, I, I, I, F, F, F, I, P, P, P, P, S, P, P]
        L.entmaxkv_sparse_attend.argtypes = [PP, P, I, P, I, P, I, P, P, I, F, F, P, P, P, P, S, P, P]
        L.entmaxkv_full_entmax_decode.argtypes = [PP, P, I, P, I, P, I, F, F, P, P, P, P, S, P, P]
        L.entmaxkv_full_softmax_decode.argtypes = [PP, P, I, P, I, P, I, F, P, P, S, P, P]
        L.entmaxkv_sparse_softmax_attend.argtypes = [PP, P, I, P, I, P, I, P, P, I, F, P, P, S, P, P]
        L.entmaxkv_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
        L.entmaxkv_workspace_size.restype = ctypes.c_size_t
        L.entmaxkv_status_string.argtypes = [I]
        L.entmaxkv_status_string.restype = ctypes.c_char_p
        L.entmaxkv_selftest_timeout.argtypes = [ctypes.c_int64, P, P]
        L.entmaxkv_sparse_attend_static.argtypes = [PP, P, I, P, I, P, I, P, P, I, F, F, P, P, P, P, P]
        L.entmaxkv_append_score_pages.argtypes = [PP, P, P, I, P, I, P, I, P, I, F, P, P, P]
        for name in SYMBOLS:
            if name not in ("entmaxkv_workspace_size", "entmaxkv_status_string"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code):
    return lib().entmaxkv_status_string(int(code)).decode()


def _check(rc, where):
    if rc != OK:
        raise EntmaxKVError(rc, where)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class _Args:
    """Checks of one call's tensors before anything is launched.  The library
    takes plain pointers, so a tensor of the wrong dtype or rank, a strided
    view, fewer elements than the sizes passed address, or memory the current
    GPU cannot reach would be read or written out of bounds; `need` checks the
    layout of each tensor as it is named and `reachable` then checks that every
    one is the current device's memory or pinned (mapped) host memory."""

    def __init__(self, where):
        self.where = where
        self.seen = []

    def fail(self, detail, code=INVALID_ARG):
        raise EntmaxKVError(code, self.where, detail)

    def need(self, t, name, dtype=None, numel=0, dims=None):
        if t is None:
            self.fail("%s is required" % name)
        if dtype is not None and t.dtype != dtype:
            self.fail("%s must be %s, not %s" % (name, dtype, t.dtype))
        if dims is not None and t.dim() != dims:
            self.fail("%s must have %d dimensions, not %d" % (name, dims, t.dim()))
        if not t.is_contiguous():
            self.fail("%s must be contiguous" % name)
        if t.numel() < numel:
            self.fail("%s holds %d elements; the call addresses %d" % (name, t.numel(), numel))
        self.seen.append((name, t))
        return t

    def reachable(self):
        dev = capturing = None
        for name, t in self.seen:
            if t.is_cuda:
                dev = torch.cuda.current_device() if dev is None else dev
                if t.get_device() != dev:
                    self.fail("%s is on cuda:%d, the current device is cuda:%d" % (name, t.get_device(), dev))
                continue
            if capturing is None:
                # the pinned-memory query is not issued while a CUDA graph is
                # being captured; the eager call before a capture checks it
                capturing = torch.cuda.is_available() and torch.cuda.is_current_stream_capturing()
            if not capturing and not t.is_pinned():
                self.fail("%s must be in device memory or pinned host memory" % name)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Pool:
    """Paged KV pool and per-page metadata, all torch device tensors.

    k_pool, v_pool [num_phys, H_kv, ps, d] (fp32 or bf16); kmin, kmax
    [num_phys, H_kv, d] same dtype; mean, m2 [num_phys, H_kv, d] fp32;
    count [num_phys] int32.
    """

    def __init__(self, k_pool, v_pool, kmin, kmax, mean, m2, count):
        a = _Args("Pool")
        if k_pool.dtype not in (torch.float32, torch.bfloat16):
            a.fail("k_pool must be float32 or bfloat16, not %s" % k_pool.dtype, UNSUPPORTED)
        a.need(k_pool, "k_pool", dims=4)
        num_phys, H_kv, ps, d = k_pool.shape
        meta = num_phys * H_kv * d
        a.need(v_pool, "v_pool", k_pool.dtype, k_pool.numel(), dims=4)
        a.need(kmin, "kmin", k_pool.dtype, meta)
        a.need(kmax, "kmax", k_pool.dtype, meta)
        a.need(mean, "mean", torch.float32, meta)
        a.need(m2, "m2", torch.float32, meta)
        a.need(count, "count", torch.int32, num_phys)
        if tuple(v_pool.shape) != tuple(k_pool.shape):
            a.fail("v_pool must have k_pool's shape")
        a.reachable()
        self.k_pool, self.v_pool = k_pool, v_pool
        self.kmin, self.kmax, self.mean, self.m2, self.count = kmin, kmax, mean, m2, count
        self.num_phys, self.H_kv, self.ps, self.d = num_phys, H_kv, ps, d
        self.dtype = BF16 if k_pool.dtype == torch.bfloat16 else F32
        self._c = CPool(k_pool.data_ptr(), v_pool.data_ptr(), kmin.data_ptr(), kmax.data_ptr(),
                        mean.data_ptr(), m2.data_ptr(), count.data_ptr(), self.num_phys, self.H_kv,
                        self.ps, self.d, self.dtype)

    @classmethod
    def allocate(cls, num_phys, H_kv, ps, d, dtype=torch.bfloat16, device="cuda"):
        kv = dict(dtype=dtype, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        return cls(torch.zeros(num_phys, H_kv, ps, d, **kv), torch.zeros(num_phys, H_kv, ps, d, **kv),
                   torch.zeros(num_phys, H_kv, d, **kv), torch.zeros(num_phys, H_kv, d, **kv),
                   torch.zeros(num_phys, H_kv, d, **f32), torch.zeros(num_phys, H_kv, d, **f32),
                   torch.zeros(num_phys, dtype=torch.int32, device=device))

    @property
    def c(self):
        return ctypes.byref(self._c)


I32, F32T = torch.int32, torch.float32


def _query(a, pool, q):
    """q [B, H_q, d] float32 with the pool's d; returns (B, H_q)."""
    a.need(q, "q", F32T, dims=3)
    if q.shape[2] != pool.d:
        a.fail("q has %d dims per head, the pool %d" % (q.shape[2], pool.d))
    return q.shape[0], q.shape[1]


def _table(a, page_table, seq_lens, B):
    """page_table [>= B, max_pages] and seq_lens [>= B], both int32; returns max_pages."""
    a.need(page_table, "page_table", I32, dims=2)
    if page_table.shape[0] < B:
        a.fail("page_table has %d rows for %d sequences" % (page_table.shape[0], B))
    a.need(seq_lens, "seq_lens", I32, B)
    return page_table.shape[1]


def _page_list(a, pool, sel, sel_count, B):
    """sel [>= B, H_kv, k_max] and sel_count [>= B * H_kv], int32; returns k_max."""
    a.need(sel, "sel", I32, dims=3)
    if sel.shape[0] < B or sel.shape[1] != pool.H_kv:
        a.fail("sel must be [B, H_kv, k_max] with B = %d and H_kv = %d" % (B, pool.H_kv))
    a.need(sel_count, "sel_count", I32, B * pool.H_kv)
    return sel.shape[2]


def _outputs(a, pool, out, tau_out, v_pages, status, B, H_q):
    a.need(out, "out", F32T, B * H_q * pool.d)
    if tau_out is not None:
        a.need(tau_out, "tau_out", F32T, B * H_q)
    if v_pages is not None:
        a.need(v_pages, "v_pages", I32, B * pool.H_kv)
    a.need(status, "status", I32, 1)


def _bytes(t):
    return t.numel() * t.element_size()


def append_metadata(pool, k_new, v_new, page_table, seq_lens, status, stream=None):
    """k_new, v_new [B, H_kv, n_new, d]; seq_lens advanced in place on the device."""
    a = _Args("append_metadata")
    a.need(k_new, "k_new", pool.k_pool.dtype, dims=4)
    B, H_kv, n_new, d = k_new.shape
    if H_kv != pool.H_kv or d != pool.d:
        a.fail("k_new must be [B, %d, n_new, %d]" % (pool.H_kv, pool.d))
    a.need(v_new, "v_new", pool.k_pool.dtype, k_new.numel(), dims=4)
    max_pages = _table(a, page_table, seq_lens, B)
    a.need(status, "status", I32, 1)
    a.reachable()
    _check(lib().entmaxkv_append_metadata(pool.c, _p(k_new), _p(v_new), n_new, _p(page_table),
                                          max_pages, _p(seq_lens), B, _p(status),
                                          _stream(stream)), a.where)


def append_score_pages(pool, k_new, v_new, q, page_table, seq_lens, scale, status, ub, stream=None):
    """append_metadata then score_pages(SCORE_BBOX) over the new lengths, in one
    call (one scoring launch where the library can fold the append into it)."""
    a = _Args("append_score_pages")
    a.need(k_new, "k_new", pool.k_pool.dtype, dims=4)
    B, H_kv, n_new, d = k_new.shape
    if H_kv != pool.H_kv or d != pool.d:
        a.fail("k_new must be [B, %d, n_new, %d]" % (pool.H_kv, pool.d))
    a.need(v_new, "v_new", pool.k_pool.dtype, k_new.numel(), dims=4)
    Bq, H_q = _query(a, pool, q)
    if Bq != B:
        a.fail("q holds %d sequences; k_new %d" % (Bq, B))
    max_pages = _table(a, page_table, seq_lens, B)
    a.need(ub, "ub", F32T, B * pool.H_kv * max_pages)
    a.need(status, "status", I32, 1)
    a.reachable()
    _check(lib().entmaxkv_append_score_pages(pool.c, _p(k_new), _p(v_new), n_new, _p(q), H_q, _p(page_table),
                                             max_pages, _p(seq_lens), B, scale, _p(ub), _p(status),
                                             _stream(stream)), a.where)


def score_pages(pool, q, page_table, seq_lens, mode, scale, status, ub=None, m=None, v=None,
                est_max=None, stream=None):
    a = _Args("score_pages")
    B, H_q = _query(a, pool, q)
    max_pages = _table(a, page_table, seq_lens, B)
    a.need(status, "status", I32, 1)
    if mode == SCORE_BBOX:
        a.need(ub, "ub", F32T, B * pool.H_kv * max_pages)
    elif mode == SCORE_GAUSS:
        for t, name in ((m, "m"), (v, "v"), (est_max, "est_max")):
            a.need(t, name, F32T, B * H_q * max_pages)
    a.reachable()
    _check(lib().entmaxkv_score_pages(pool.c, _p(q), H_q, _p(page_table), max_pages,
                                      _p(seq_lens), B, mode, scale, _p(ub), _p(m), _p(v), _p(est_max),
                                      _p(status), _stream(stream)), a.where)


def select(mode, seq_lens, ps, H_q, H_kv, max_pages, k_max, sel, sel_count, status, ub=None, m=None,
           v=None, est_max=None, budget=-1, budget_frac=0.0, alpha=1.5, delta=0.0, tau_hat=None,
           stream=None):
    a = _Args("select")
    a.need(seq_lens, "seq_lens", I32, dims=1)
    B = seq_lens.shape[0]
    a.need(sel, "sel", I32, B * H_kv * k_max)
    a.need(sel_count, "sel_count", I32, B * H_kv)
    a.need(status, "status", I32, 1)
    if mode == SELECT_TOPK:
        a.need(ub, "ub", F32T, B * H_kv * max_pages)
    elif mode == SELECT_GAUSS:
        for t, name in ((m, "m"), (v, "v"), (est_max, "est_max")):
            a.need(t, name, F32T, B * H_q * max_pages)
        a.need(tau_hat, "tau_hat", F32T, B * H_q)
    a.reachable()
    _check(lib().entmaxkv_select(mode, _p(ub), _p(m), _p(v), _p(est_max), _p(seq_lens), ps, B, H_q,
                                 H_kv, max_pages, budget, budget_frac, alpha, delta, k_max, _p(sel),
                                 _p(sel_count), _p(tau_hat), None, 0, _p(status), _stream(stream)), a.where)


def workspace_size(op, B, H_q, H_kv, max_pages, k_max, ps, d):
    return int(lib().entmaxkv_workspace_size(op, B, H_q, H_kv, max_pages, k_max, ps, d))


def sparse_attend(pool, q, page_table, seq_lens, sel, sel_count, alpha, scale, out, workspace, status,
                  tau_out=None, v_pages=None, stream=None):
    a = _Args("sparse_attend")
    B, H_q = _query(a, pool, q)
    max_pages = _table(a, page_table, seq_lens, B)
    k_max = _page_list(a, pool, sel, sel_count, B)
    _outputs(a, pool, out, tau_out, v_pages, status, B, H_q)
    a.need(workspace, "workspace")
    a.reachable()
    _check(lib().entmaxkv_sparse_attend(pool.c, _p(q), H_q, _p(page_table), max_pages,
                                        _p(seq_lens), B, _p(sel), _p(sel_count), k_max, alpha,
                                        scale, _p(out), _p(tau_out), _p(v_pages), _p(workspace),
                                        _bytes(workspace), _p(status), _stream(stream)), a.where)


def sparse_attend_static(pool, q, page_table, seq_lens, sel, sel_count, alpha, scale, out, status,
                         tau_out=None, v_pages=None, stream=None):
    """sparse_attend with the library's built-in scratch buffer (no workspace)."""
    a = _Args("sparse_attend_static")
    B, H_q = _query(a, pool, q)
    max_pages = _table(a, page_table, seq_lens, B)
    k_max = _page_list(a, pool, sel, sel_count, B)
    _outputs(a, pool, out, tau_out, v_pages, status, B, H_q)
    a.reachable()
    _check(lib().entmaxkv_sparse_attend_static(pool.c, _p(q), H_q, _p(page_table), max_pages,
                                               _p(seq_lens), B, _p(sel), _p(sel_count), k_max, alpha,
                                               scale, _p(out), _p(tau_out), _p(v_pages), _p(status),
                                               _stream(stream)), a.where)


def full_entmax_decode(pool, q, page_table, seq_lens, alpha, scale, out, workspace, status,
                       tau_out=None, v_pages=None, stream=None):
    a = _Args("full_entmax_decode")
    B, H_q = _query(a, pool, q)
    max_pages = _table(a, page_table, seq_lens, B)
    _outputs(a, pool, out, tau_out, v_pages, status, B, H_q)
    a.need(workspace, "workspace")
    a.reachable()
    _check(lib().entmaxkv_full_entmax_decode(pool.c, _p(q), H_q, _p(page_table), max_pages,
                                             _p(seq_lens), B, alpha, scale, _p(out), _p(tau_out), _p(v_pages),
                                             _p(workspace), _bytes(workspace), _p(status), _stream(stream)),
           a.where)


def full_softmax_decode(pool, q, page_table, seq_lens, scale, out, workspace, status, stream=None):
    a = _Args("full_softmax_decode")
    B, H_q = _query(a, pool, q)
    max_pages = _table(a, page_table, seq_lens, B)
    _outputs(a, pool, out, None, None, status, B, H_q)
    a.need(workspace, "workspace")
    a.reachable()
    _check(lib().entmaxkv_full_softmax_decode(pool.c, _p(q), H_q, _p(page_table), max_pages,
                                              _p(seq_lens), B, scale, _p(out), _p(workspace),
                                              _bytes(workspace), _p(status), _stream(stream)), a.where)


def sparse_softmax_attend(pool, q, page_table, seq_lens, sel, sel_count, scale, out, workspace, status,
                          stream=None):
    """Softmax attention over the listed pages (workspace: OP_SPARSE_SOFTMAX)."""
    a = _Args("sparse_softmax_attend")
    B, H_q = _query(a, pool, q)
    max_pages = _table(a, page_table, seq_lens, B)
    k_max = _page_list(a, pool, sel, sel_count, B)
    _outputs(a, pool, out, None, None, status, B, H_q)
    a.need(workspace, "workspace")
    a.reachable()
    _check(lib().entmaxkv_sparse_softmax_attend(pool.c, _p(q), H_q, _p(page_table), max_pages,
                                                _p(seq_lens), B, _p(sel), _p(sel_count), k_max, scale,
                                                _p(out), _p(workspace), _bytes(workspace),
                                                _p(status), _stream(stream)), a.where)


def selftest_timeout(limit_ns, status, stream=None):
    a = _Args("selftest_timeout")
    a.need(status, "status", I32, 1)
    a.reachable()
    _check(lib().entmaxkv_selftest_timeout(int(limit_ns), _p(status), _stream(stream)), a.where)
