"""Thin ctypes binding over the EntmaxKV C ABI (include/entmaxkv.h).

Argument marshalling only: every function below passes torch tensors' device
pointers, sizes and the current CUDA stream to the entry point of the same
name and raises on a non-zero host status.  All work runs in the CUDA library;
there is no other implementation to fall back to -- if the shared library is
missing the first call raises.
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
    "entmaxkv_sparse_softmax_attend",
)


class EntmaxKVError(RuntimeError):
    def __init__(self, code, where):
        super().__init__("%s: %s (status %d)" % (where, status_string(code), code))
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
        self.k_pool, self.v_pool = k_pool, v_pool
        self.kmin, self.kmax, self.mean, self.m2, self.count = kmin, kmax, mean, m2, count
        self.num_phys, self.H_kv, self.ps, self.d = k_pool.shape
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


def append_metadata(pool, k_new, v_new, page_table, seq_lens, status, stream=None):
    """k_new, v_new [B, H_kv, n_new, d]; seq_lens advanced in place on the device."""
    B, _, n_new, _ = k_new.shape
    _check(lib().entmaxkv_append_metadata(pool.c, _p(k_new), _p(v_new), n_new, _p(page_table),
                                          page_table.shape[1], _p(seq_lens), B, _p(status),
                                          _stream(stream)), "append_metadata")


def score_pages(pool, q, page_table, seq_lens, mode, scale, status, ub=None, m=None, v=None,
                est_max=None, stream=None):
    B, H_q, _ = q.shape
    _check(lib().entmaxkv_score_pages(pool.c, _p(q), H_q, _p(page_table), page_table.shape[1],
                                      _p(seq_lens), B, mode, scale, _p(ub), _p(m), _p(v), _p(est_max),
                                      _p(status), _stream(stream)), "score_pages")


def select(mode, seq_lens, ps, H_q, H_kv, max_pages, k_max, sel, sel_count, status, ub=None, m=None,
           v=None, est_max=None, budget=-1, budget_frac=0.0, alpha=1.5, delta=0.0, tau_hat=None,
           stream=None):
    B = seq_lens.shape[0]
    _check(lib().entmaxkv_select(mode, _p(ub), _p(m), _p(v), _p(est_max), _p(seq_lens), ps, B, H_q,
                                 H_kv, max_pages, budget, budget_frac, alpha, delta, k_max, _p(sel),
                                 _p(sel_count), _p(tau_hat), None, 0, _p(status), _stream(stream)),
           "select")


def workspace_size(op, B, H_q, H_kv, max_pages, k_max, ps, d):
    return int(lib().entmaxkv_workspace_size(op, B, H_q, H_kv, max_pages, k_max, ps, d))


def sparse_attend(pool, q, page_table, seq_lens, sel, sel_count, alpha, scale, out, workspace, status,
                  tau_out=None, v_pages=None, stream=None):
    B, H_q, _ = q.shape
    _check(lib().entmaxkv_sparse_attend(pool.c, _p(q), H_q, _p(page_table), page_table.shape[1],
                                        _p(seq_lens), B, _p(sel), _p(sel_count), sel.shape[2], alpha,
                                        scale, _p(out), _p(tau_out), _p(v_pages), _p(workspace),
                                        workspace.numel() * workspace.element_size(), _p(status),
                                        _stream(stream)), "sparse_attend")


def sparse_attend_static(pool, q, page_table, seq_lens, sel, sel_count, alpha, scale, out, status,
                         tau_out=None, v_pages=None, stream=None):
    """sparse_attend with the library's built-in scratch buffer (no workspace)."""
    B, H_q, _ = q.shape
    _check(lib().entmaxkv_sparse_attend_static(pool.c, _p(q), H_q, _p(page_table), page_table.shape[1],
                                               _p(seq_lens), B, _p(sel), _p(sel_count), sel.shape[2], alpha,
                                               scale, _p(out), _p(tau_out), _p(v_pages), _p(status),
                                               _stream(stream)), "sparse_attend_static")


def full_entmax_decode(pool, q, page_table, seq_lens, alpha, scale, out, workspace, status,
                       tau_out=None, v_pages=None, stream=None):
    B, H_q, _ = q.shape
    _check(lib().entmaxkv_full_entmax_decode(pool.c, _p(q), H_q, _p(page_table), page_table.shape[1],
                                             _p(seq_lens), B, alpha, scale, _p(out), _p(tau_out), _p(v_pages),
                                             _p(workspace), workspace.numel() * workspace.element_size(),
                                             _p(status), _stream(stream)), "full_entmax_decode")


def full_softmax_decode(pool, q, page_table, seq_lens, scale, out, workspace, status, stream=None):
    B, H_q, _ = q.shape
    _check(lib().entmaxkv_full_softmax_decode(pool.c, _p(q), H_q, _p(page_table), page_table.shape[1],
                                              _p(seq_lens), B, scale, _p(out), _p(workspace),
                                              workspace.numel() * workspace.element_size(), _p(status),
                                              _stream(stream)), "full_softmax_decode")


def sparse_softmax_attend(pool, q, page_table, seq_lens, sel, sel_count, scale, out, workspace, status,
                          stream=None):
    """Softmax attention over the listed pages (workspace: OP_SPARSE_SOFTMAX)."""
    B, H_q, _ = q.shape
    _check(lib().entmaxkv_sparse_softmax_attend(pool.c, _p(q), H_q, _p(page_table), page_table.shape[1],
                                                _p(seq_lens), B, _p(sel), _p(sel_count), sel.shape[2], scale,
                                                _p(out), _p(workspace), workspace.numel() * workspace.element_size(),
                                                _p(status), _stream(stream)), "sparse_softmax_attend")


def selftest_timeout(limit_ns, status, stream=None):
    _check(lib().entmaxkv_selftest_timeout(int(limit_ns), _p(status), _stream(stream)), "selftest_timeout")
