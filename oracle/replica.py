"""ctypes shim over replica_f32.c (test infrastructure only).

The fp32 canonical-order replicas decide page selection in the same precision
and order as the GPU kernels must (see the comment at the top of
replica_f32.c for the exact operation order: Welford metadata in token order;
dot products over d as 8 consecutive slices of serial fmaf chains combined by a
fixed pairwise tree).  ``build()`` compiles the C file
with gcc; it is called lazily on first use.
"""

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "replica_f32.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_OUT_DIR, "libreplica_f32.so")
_lib = None


def build(force=False):
    """Compile replica_f32.c into oracle/_build/libreplica_f32.so."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp.%d" % os.getpid()
    subprocess.check_call([
        "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
        "-fno-fast-math", "-fno-unsafe-math-optimizations", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f32p = ctypes.POINTER(ctypes.c_float)
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.replica_page_meta.argtypes = [f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                          f32p, f32p, f32p, f32p, i32p]
        lib.replica_bound.argtypes = [f32p, ctypes.c_int, ctypes.c_int, f32p, f32p,
                                      ctypes.c_int64, ctypes.c_float, f32p, f32p]
        lib.replica_gauss.argtypes = [f32p, ctypes.c_int, ctypes.c_int, f32p, f32p, i32p,
                                      ctypes.c_int64, ctypes.c_float, f32p, f32p, f32p, f32p]
        for fn in (lib.replica_page_meta, lib.replica_bound, lib.replica_gauss):
            fn.restype = None
        _lib = lib
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a, ct=ctypes.c_float):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def page_meta(keys, ps):
    """fp32 Welford metadata of the pages of one (sequence, kv-head).

    keys: [L, d] (fp32, or bf16 values already widened).  Returns dict of
    kmin, kmax, mean, m2 ([P, d] float32) and count ([P] int32).
    """
    keys = _f32(keys)
    L, d = keys.shape
    P = (L + ps - 1) // ps
    out = {k: np.zeros((P, d), dtype=np.float32) for k in ("kmin", "kmax", "mean", "m2")}
    out["count"] = np.zeros(P, dtype=np.int32)
    _load().replica_page_meta(_ptr(keys), L, d, ps, _ptr(out["kmin"]), _ptr(out["kmax"]),
                              _ptr(out["mean"]), _ptr(out["m2"]),
                              _ptr(out["count"], ctypes.c_int32))
    return out


def bound(q, kmin, kmax, scale):
    """(ub [G, P], ubg [P]) fp32 bounding-box bounds in the canonical order."""
    q = _f32(q)
    kmin = _f32(kmin)
    kmax = _f32(kmax)
    G, d = q.shape
    if d % 8:
        raise ValueError("the canonical order splits d into 8 slices: d must be a multiple of 8")
    P = kmin.shape[0]
    ub = np.zeros((G, P), dtype=np.float32)
    ubg = np.zeros(P, dtype=np.float32)
    _load().replica_bound(_ptr(q), G, d, _ptr(kmin), _ptr(kmax), P,
                          ctypes.c_float(scale), _ptr(ub), _ptr(ubg))
    return ub, ubg


def z_table_f32(ps):
    """fp32 rounding of z_n = sqrt(2 ln n) (n >= 2), z_0 = z_1 = 0."""
    import math
    z = np.zeros(ps + 1, dtype=np.float32)
    for n in range(2, ps + 1):
        z[n] = np.float32(math.sqrt(2.0 * math.log(n)))
    return z


def gauss(q, mean, m2, count, scale, ps):
    """(m, v, est) [G, P] fp32 Gaussian page estimates in the canonical order."""
    q = _f32(q)
    mean = _f32(mean)
    m2 = _f32(m2)
    count = np.ascontiguousarray(count, dtype=np.int32)
    if count.size and (count.min() < 1 or count.max() > ps):
        raise ValueError("page counts must lie in [1, ps]")
    G, d = q.shape
    if d % 8:
        raise ValueError("the canonical order splits d into 8 slices: d must be a multiple of 8")
    P = mean.shape[0]
    z = z_table_f32(ps)
    m = np.zeros((G, P), dtype=np.float32)
    v = np.zeros((G, P), dtype=np.float32)
    est = np.zeros((G, P), dtype=np.float32)
    _load().replica_gauss(_ptr(q), G, d, _ptr(mean), _ptr(m2), _ptr(count, ctypes.c_int32),
                          P, ctypes.c_float(scale), _ptr(z), _ptr(m), _ptr(v), _ptr(est))
    return m, v, est
