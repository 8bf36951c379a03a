"""Decode-step driver: buffers plus the ordered C-ABI calls of one EntmaxKV step.

    append (optional) -> score_pages -> select -> sparse_attend

Host orchestration only -- it allocates device buffers with torch once and
issues the library calls in order on one stream; every step of the path runs
in the CUDA library.
"""
import math

import torch

from . import binding as B
from .workloads import Workload


def build_pool(wl: Workload, device="cuda", status=None):
    """Allocate the pool of a workload and fill it sequence by sequence with
    entmaxkv_append_metadata (whole-sequence appends build every page).
    Returns (pool, seq_lens tensor on device)."""
    cfg = wl.cfg
    pool = B.Pool.allocate(wl.num_phys, cfg.H_kv, cfg.ps, cfg.d, cfg.dtype, device)
    seq_lens = torch.zeros(cfg.B, dtype=torch.int32, device=device)
    st = torch.zeros(1, dtype=torch.int32, device=device) if status is None else status
    pt = wl.page_table.to(device)
    for b in range(cfg.B):
        k, v = wl.sequence(b)
        k = k.to(device).unsqueeze(0).contiguous()
        v = v.to(device).unsqueeze(0).contiguous()
        B.append_metadata(pool, k, v, pt[b:b + 1], seq_lens[b:b + 1], st)
        del k, v
    if status is None:
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise B.EntmaxKVError(int(st.item()), "build_pool")
    return pool, seq_lens


class DecodeStep:
    """One decode step of a configuration: scores, selects and attends.

    mode "topk" (budget pages or budget_frac) or "gauss" (alpha, delta).
    out: optional float32 [B][H_q][d] result buffer, on the device or in
    pinned host memory.
    """

    def __init__(self, pool, page_table, seq_lens, H_q, mode="topk", budget=-1, budget_frac=0.0,
                 alpha=1.5, delta=0.5, extra_pages=0, out=None):
        self.pool, self.page_table, self.seq_lens = pool, page_table, seq_lens
        self.B = seq_lens.shape[0]
        self.H_q, self.H_kv = H_q, pool.H_kv
        self.max_pages = page_table.shape[1]
        self.mode, self.budget, self.budget_frac = mode, budget, budget_frac
        self.alpha, self.delta = alpha, delta
        self.scale = 1.0 / math.sqrt(pool.d)
        dev = pool.k_pool.device
        f32 = dict(dtype=torch.float32, device=dev)
        i32 = dict(dtype=torch.int32, device=dev)
        if mode == "topk":
            self.k_max = budget if budget >= 0 else int(math.ceil(float(torch.tensor(budget_frac,
                                                                                       dtype=torch.float32))
                                                                   * self.max_pages))
            self.k_max = max(1, self.k_max)
            self.ub = torch.empty(self.B, self.H_kv, self.max_pages, **f32)
            self.m = self.v = self.est = self.tau_hat = None
        else:
            self.k_max = self.max_pages
            self.ub = None
            self.m = torch.empty(self.B, H_q, self.max_pages, **f32)
            self.v = torch.empty_like(self.m)
            self.est = torch.empty_like(self.m)
            self.tau_hat = torch.empty(self.B, H_q, **f32)
        self.sel = torch.empty(self.B, self.H_kv, self.k_max, **i32)
        self.sel_count = torch.empty(self.B, self.H_kv, **i32)
        # out may be pinned host memory (mapped into the device's address space):
        # the attention kernels then store the result straight to the host
        self.out = torch.empty(self.B, H_q, pool.d, **f32) if out is None else out
        self.tau = torch.empty(self.B, H_q, **f32)
        ws = B.workspace_size(B.OP_SPARSE_ATTEND, self.B, H_q, self.H_kv, self.max_pages, self.k_max,
                              pool.ps, pool.d)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, **i32)
        self.v_pages = torch.zeros(self.B, self.H_kv, **i32)     # value pages loaded, accumulated

    def score(self, q, stream=None):
        if self.mode == "topk":
            B.score_pages(self.pool, q, self.page_table, self.seq_lens, B.SCORE_BBOX, self.scale, self.status,
                          ub=self.ub, stream=stream)
        else:
            B.score_pages(self.pool, q, self.page_table, self.seq_lens, B.SCORE_GAUSS, self.scale, self.status,
                          m=self.m, v=self.v, est_max=self.est, stream=stream)

    def choose(self, stream=None):
        if self.mode == "topk":
            B.select(B.SELECT_TOPK, self.seq_lens, self.pool.ps, self.H_q, self.H_kv, self.max_pages, self.k_max,
                     self.sel, self.sel_count, self.status, ub=self.ub, budget=self.budget,
                     budget_frac=self.budget_frac, stream=stream)
        else:
            B.select(B.SELECT_GAUSS, self.seq_lens, self.pool.ps, self.H_q, self.H_kv, self.max_pages,
                     self.k_max, self.sel, self.sel_count, self.status, m=self.m, v=self.v, est_max=self.est,
                     alpha=self.alpha, delta=self.delta, tau_hat=self.tau_hat, stream=stream)

    def attend(self, q, stream=None):
        B.sparse_attend(self.pool, q, self.page_table, self.seq_lens, self.sel, self.sel_count, self.alpha,
                        self.scale, self.out, self.workspace, self.status, tau_out=self.tau,
                        v_pages=self.v_pages, stream=stream)

    def append_score(self, q, k_new, v_new, stream=None):
        """Append (k_new, v_new) [B, H_kv, n, d], then score over the new lengths
        (top-k mode: one library call, which can fold the append into the
        scoring launch)."""
        if self.mode == "topk":
            B.append_score_pages(self.pool, k_new, v_new, q, self.page_table, self.seq_lens, self.scale,
                                 self.status, self.ub, stream=stream)
        else:
            B.append_metadata(self.pool, k_new, v_new, self.page_table, self.seq_lens, self.status, stream=stream)
            self.score(q, stream)

    def __call__(self, q, k_new=None, v_new=None, stream=None):
        """One step; appends (k_new, v_new) [B, H_kv, 1, d] first when given."""
        if k_new is not None:
            self.append_score(q, k_new, v_new, stream)
        else:
            self.score(q, stream)
        self.choose(stream)
        self.attend(q, stream)
        return self.out

    def check(self):
        torch.cuda.synchronize()
        code = int(self.status.item())
        if code:
            raise B.EntmaxKVError(code, "decode step (device status)")


class _CudaRT:
    """Event-record nodes inside a captured graph (cudaEventRecordWithFlags with
    cudaEventRecordExternal) so stage boundaries can be timed during replay."""

    def __init__(self):
        import ctypes
        self.ct = ctypes
        self.rt = ctypes.CDLL("libcudart.so.12")
        self.rt.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_uint]
        self.rt.cudaEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
        self.rt.cudaEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_void_p, ctypes.c_void_p]
        self.rt.cudaEventDestroy.argtypes = [ctypes.c_void_p]

    def event(self):
        e = self.ct.c_void_p()
        if self.rt.cudaEventCreateWithFlags(self.ct.byref(e), 0) != 0:
            raise RuntimeError("cudaEventCreateWithFlags failed")
        return e

    def record_node(self, e, stream):
        rc = self.rt.cudaEventRecordWithFlags(e, self.ct.c_void_p(stream.cuda_stream), 1)
        if rc != 0:
            raise RuntimeError("cudaEventRecordWithFlags failed (%d)" % rc)

    def elapsed_ms(self, a, b):
        ms = self.ct.c_float()
        rc = self.rt.cudaEventElapsedTime(self.ct.byref(ms), a, b)
        return None if rc != 0 else ms.value


class GraphedStep:
    """A DecodeStep captured once into a CUDA graph.

    The step's inputs live in static device buffers (q, k, v): copy the new
    query and token into them, then replay().  With stage_events=True the
    graph also records an event node between stages; stage_us() returns the
    last replay's per-stage durations (append, score, select, attend) in us.
    In top-k mode the append is part of the scoring call (append_score), so
    the append stage is empty and the score stage holds both.
    """

    STAGES = ("append", "score", "select", "attend")

    def __init__(self, step: DecodeStep, append=True, stage_events=True):
        self.step = step
        pool = step.pool
        dev = pool.k_pool.device
        # q, k and v are views of one device buffer, so a step's inputs can
        # arrive in a single host-to-device copy (pack_host / inputs)
        elt = pool.k_pool.element_size()
        nq = step.B * step.H_q * pool.d * 4
        nk = step.B * step.H_kv * pool.d * elt
        al = lambda x: (x + 255) // 256 * 256
        self._off = (0, al(nq), al(nq) + al(nk))
        self._len = (nq, nk, nk)
        self.inputs = torch.zeros(al(nq) + 2 * al(nk), dtype=torch.uint8, device=dev)
        self.q = self._view(self.inputs, 0).view(torch.float32).view(step.B, step.H_q, pool.d)
        self.k = self._view(self.inputs, 1).view(pool.k_pool.dtype).view(step.B, step.H_kv, 1, pool.d)
        self.v = self._view(self.inputs, 2).view(pool.k_pool.dtype).view(step.B, step.H_kv, 1, pool.d)
        self.append = append
        self.rt = _CudaRT() if stage_events else None
        self.ev = [self.rt.event() for _ in range(5)] if stage_events else None
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):          # warm-up outside capture (no append)
            step.score(self.q)
            step.choose()
            step.attend(self.q)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            cs = torch.cuda.current_stream()
            self._mark(0, cs)
            if append and step.mode != "topk":
                B.append_metadata(pool, self.k, self.v, step.page_table, step.seq_lens, step.status)
            self._mark(1, cs)
            if append and step.mode == "topk":
                step.append_score(self.q, self.k, self.v)
            else:
                step.score(self.q)
            self._mark(2, cs)
            step.choose()
            self._mark(3, cs)
            step.attend(self.q)
            self._mark(4, cs)

    def _view(self, buf, i):
        return buf[self._off[i]:self._off[i] + self._len[i]]

    def pack_host(self, k, v, q):
        """Pinned host buffer laid out like `inputs` holding (k, v, q) of one
        step: copy it into `inputs` with one copy, then replay()."""
        h = torch.zeros(self.inputs.numel(), dtype=torch.uint8).pin_memory()
        for i, t in ((0, q), (1, k), (2, v)):
            src = t.detach().to("cpu").contiguous().reshape(-1).view(torch.uint8)
            self._view(h, i).copy_(src)
        return h

    def _mark(self, i, stream):
        if self.ev is not None:
            self.rt.record_node(self.ev[i], stream)

    def replay(self):
        self.graph.replay()
        return self.step.out

    def stage_us(self):
        if self.ev is None:
            return None
        out = {}
        for i, name in enumerate(self.STAGES):
            ms = self.rt.elapsed_ms(self.ev[i], self.ev[i + 1])
            out[name] = None if ms is None else ms * 1e3
        return out
