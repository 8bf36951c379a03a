"""Benchmark: one EntmaxKV decode step at 1M-token context on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

A step is the whole decode path on one batch: append the step's token (KV
write + page metadata), score every page (bounding-box bound), select the top
1/64 of pages per kv head, and run exact 1.5-entmax attention over the
selected pages.  Workload: B=1 sequence of 2^20 tokens per GPU, 32 query / 8
kv heads, head dim 128, pages of 64, bf16 cache (synthetic clustered keys with
planted tokens).  L2 is flushed between timed steps, outside the per-step
CUDA events: a 256 MiB buffer is written, then a second 256 MiB buffer is
read, so that the written lines are back in HBM before the step starts.  Rank
0 prints one JSON line.

--impl reference times the CPU oracle on the host cores instead (rank 0 only).
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse entmax decode µs/step @1M ctx; achieved HBM GB/s vs 8 TB/s roofline"
# DRAM bytes the scoring kernel read per (page, kv head) metadata row in an ncu
# capture of the 2^18-token case (16,865,024 bytes for 4097 pages x 8 heads);
# scaled by rows to the bench launch.  Must be re-measured when the scoring
# kernel changes.
SCORE_DRAM_BYTES_PER_ROW = 16865024 / (4097 * 8)
# DRAM bytes (read + write) of one fused attention launch of the 2^20-token
# top-k 1/64 workload in an ncu capture (the first graph replay); reported as
# that launch's traffic beside the mean algorithmic bytes.  Must be re-measured
# when the attention kernel changes.
ATTEND_DRAM_BYTES_1M = 37660000 + 50940   # 37.66 MB read, 50.94 KB written (ncu rounding)
HBM_NOMINAL_GBS = 8000.0
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
MiB = 1 << 20


class L2Flush:
    """Evicts the step's data from L2 between timed steps: a 256 MiB write,
    then a read of another 256 MiB buffer, so that the write's dirty lines
    drain to HBM here rather than inside the next step (L2 is 126 MB); no
    host synchronisation."""

    def __init__(self):
        self.w = torch.empty(256 * MiB, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(256 * MiB, dtype=torch.uint8, device="cuda")
        self.sink = torch.zeros((), dtype=torch.int64, device="cuda")

    def __call__(self, i):
        self.w.fill_(i & 0xFF)
        torch.sum(self.r, dim=0, dtype=torch.int64, out=self.sink)

    def fill_(self, v):
        self(v)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--context", type=int, default=1 << 20, help="tokens per sequence (default 2^20)")
    ap.add_argument("--no-baselines", action="store_true", help="skip the full-cache and Gaussian timings")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline leg")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration legs (configurations 2, 3 and 5 at their sizes)")
    ap.add_argument("--replay-only", choices=["topk", "gauss"], default=None,
                    help="build the workload, capture that step as a graph and replay it --steps times "
                         "without timing (a short program for profiler launch lists)")
    ap.add_argument("--oracle-leg", action="store_true",
                    help="time the CPU oracle on this host's cores and print one JSON line (no GPU)")
    ap.add_argument("--leg-seconds", type=float, default=8.0,
                    help="time budget of each part of the oracle leg (seconds)")
    ap.add_argument("--selector-sweep", action="store_true",
                    help="time the top-k 1/64 and the Gaussian (Delta 0.5) steps at 2^18, 2^19 and 2^20 tokens "
                         "and print one JSON line per (length, selector)")
    return ap.parse_args()


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------- distributed
def dist_init(n, backend="nccl"):
    """One process per GPU under torchrun.  The native arm reduces its timings
    over NCCL; the reference arm (host cores only) needs no GPU and uses gloo."""
    import datetime
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    timeout = datetime.timedelta(seconds=120)
    if world > 1 and backend == "nccl":
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
    elif world > 1:
        torch.distributed.init_process_group(backend, timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device="cuda"):
    """The slowest rank's value (timings are reported as the max over ranks)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class Clocks:
    """nvidia-smi samples of SM clock and throttle reasons during a timed region.

    The sampler starts `lead_s` before the region (nvidia-smi takes a moment to
    come up) and each sample carries nvidia-smi's own timestamp, so the summary
    keeps the samples taken between entering and leaving the region (all of
    them if the clocks of the two cannot be compared).  The GPU is named by its
    PCI address, which nvidia-smi and CUDA agree on whatever device indices a
    process sees; the CUDA index is the fallback."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    TS_FORMAT = "%Y/%m/%d %H:%M:%S.%f"

    def __init__(self, device_index, interval_ms=50, lead_s=0.5, smi="nvidia-smi"):
        self.dev = device_index
        self.interval_ms = interval_ms
        self.lead_s = lead_s
        self.smi = smi
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def target(self):
        """nvidia-smi's -i argument for CUDA device `dev`."""
        try:
            p = torch.cuda.get_device_properties(self.dev)
            pci = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            r = subprocess.run([self.smi, "-i", pci, "--query-gpu=index", "--format=csv,noheader"],
                               capture_output=True, text=True, timeout=20)
            if r.returncode == 0 and r.stdout.strip():
                return pci
        except Exception:
            pass
        return str(self.dev)

    def __enter__(self):
        import datetime
        try:
            self.proc = subprocess.Popen(
                [self.smi, "-i", self.target(), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", str(self.interval_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(self.lead_s)
        except Exception:
            self.proc = None
        self.t0 = datetime.datetime.now()
        return self

    def __exit__(self, *a):
        import datetime
        import signal
        self.t1 = datetime.datetime.now()
        self.lines = []
        if self.proc is not None:
            time.sleep(self.interval_ms / 1000.0)          # one more sample after the region
            out = ""
            try:
                self.proc.send_signal(signal.SIGINT)       # nvidia-smi's own way to end a loop
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                try:
                    out, _ = self.proc.communicate(timeout=5)
                except Exception:
                    out = ""
            self.lines = [l for l in (out or "").splitlines() if l.strip()]

    def summary(self):
        import datetime
        rows = []
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 10:
                continue
            try:
                sm, mx = float(f[2]), float(f[3])
            except ValueError:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], self.TS_FORMAT)
            except ValueError:
                ts = None
            rows.append((ts, sm, mx, [n for n, v in zip(self.REASONS, f[6:10]) if v.lower() == "active"]))
        window = "timed region"
        stamped = [r for r in rows if r[0] is not None and self.t0 is not None]
        inside = [r for r in stamped if self.t0 <= r[0] <= self.t1]
        if not inside and stamped:
            gap = lambda r: (self.t0 - r[0]) if r[0] < self.t0 else (r[0] - self.t1)
            inside, window = [min(stamped, key=gap)], "nearest sample (the region was shorter than the interval)"
        elif not inside:
            inside, window = rows, ("all samples (timestamps not readable)" if rows else "no samples")
        reasons = sorted({n for r in inside for n in r[3]})
        return {"sm_mhz": statistics.median(r[1] for r in inside) if inside else None,
                "sm_max_mhz": inside[-1][2] if inside else None, "reasons": reasons,
                "samples": len(inside), "window": window}


# ---------------------------------------------------------------- workload
def make_workload(context, rank, device="cuda", appends=256):
    """Rank r decodes its own independent sequence (seed offset by r); the page
    table leaves room for `appends` decode tokens."""
    import dataclasses
    from sparse_long_context_min_b200 import workloads
    cfg = workloads.config(4)
    cfg = dataclasses.replace(cfg, lengths=[context], seed=cfg.seed + 100 * rank, decode_steps=appends)
    return workloads.Workload(cfg, device=device)


def workload_name(context):
    """The bench workload, named the same way by both arms."""
    head = "million-token decode" if context == 1 << 20 else "decode at %d tokens" % context
    return ("%s: B=1 x %d tokens per GPU, 32/8 heads, d=128, page 64, bf16 KV, alpha=1.5, top-k 1/64 of pages, "
            "append 1 token per step" % (head, context))


def algorithmic_bytes(cfg, k_pages, v_pages, mode):
    """Bytes one step must move: metadata of every page, keys of the selected
    pages, values of the selected pages that hold weight, the appended token
    with its metadata row, the page table and the outputs."""
    d, ps, Hkv, Hq, B = cfg.d, cfg.ps, cfg.H_kv, cfg.H_q, cfg.B
    P = sum(cfg.pages(b) for b in range(B))
    elt = 2 if cfg.dtype == torch.bfloat16 else 4
    if mode == "topk":
        meta = P * Hkv * d * 2 * elt + B * Hkv * P * 4            # kmin, kmax read; ub written
    else:
        meta = P * Hkv * d * 2 * 4 + 3 * B * Hq * P * 4           # mean, m2 read; m, v, est written
    kv = (k_pages + v_pages) * ps * d * elt                       # K of selected, V of weighted pages
    append = B * Hkv * d * (2 * elt + 2 * (2 * elt + 2 * 4))      # token write + metadata row r/w
    table = B * P * 4
    out = B * Hq * d * 4
    return {"score": meta + table, "attend": kv, "total": meta + kv + append + table + out}


def score_bytes(cfg, mode):
    return algorithmic_bytes(cfg, 0, 0, mode)["score"]


N_LAUNCH = 4   # per step: scoring with the token append, the length advance, top-k, fused attention


def roofline_entry(kernel, nbytes, us, peak, traffic=None, note=None):
    """{bound, achieved, peak, unit, frac, traffic} of a kernel moving `nbytes`
    algorithmic bytes in `us` microseconds, against the copy peak (GB/s)."""
    peak_gbs, peak_kind = peak
    achieved = nbytes / (us * 1e-6) / 1e9
    e = {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak_gbs, "peak_kind": peak_kind,
         "unit": "GB/s", "frac": round(achieved / peak_gbs, 4), "frac_of_8tbs": round(achieved / HBM_NOMINAL_GBS, 4),
         "traffic": traffic, "bytes_per_launch": nbytes}
    if note:
        e["traffic_note"] = note
    return e


def native_line(cfg, world, K, W, mean_us, best_us, median_us, score_us, stage, sel_total, v_total, extra, e2e,
                clk, cpu, peak, attend_us):
    """The native arm's JSON line from the measured numbers (times are the
    max over ranks; e2e = (us per step, H2D bytes, D2H bytes); peak = (GB/s,
    "measured" or "fallback"))."""
    by = algorithmic_bytes(cfg, sel_total, v_total, "topk")
    peak_gbs, peak_kind = peak
    e2e_us, h2d, d2h = e2e
    step_gbs = by["total"] / (mean_us * 1e-6) / 1e9
    line = {
        "metric": METRIC,
        "value": round(mean_us, 2),
        "unit": "us/step",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(mean_us / 1e3, 5),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded clustered-page keys, planted tokens; no dataset)",
        "config": {
            "workload": workload_name(cfg.lengths[0]),
            "global_batch": world,
            "seq_len": cfg.lengths[0],
            "parallelism": "replicas: one independent sequence per GPU" if world > 1 else "single GPU",
            "l2": "flushed between steps outside the step events (256 MiB written, then another 256 MiB read)",
            "selected_pages_per_step": round(sel_total, 1),
            "value_pages_loaded_per_step": round(v_total, 1),
            "algorithmic_bytes_per_step": by["total"],
            "achieved_gbs_step": round(step_gbs, 1),
            "frac_of_8tbs": round(step_gbs / HBM_NOMINAL_GBS, 4),
            "frac_of_measured_hbm": round(step_gbs / peak_gbs, 4),
            "step_us_best": round(best_us, 2),
            "step_us_median": round(median_us, 2),
            "stage_us": {k: round(v, 2) for k, v in stage.items()},
            "stage_note": "stage_us from a graph with event nodes between stages (no overlap across them)",
            **extra,
        },
        "roofline_score": roofline_entry(
            "score_box16_kernel (entmaxkv_append_score_pages, bbox, bf16)", by["score"], score_us, peak,
            round(SCORE_DRAM_BYTES_PER_ROW * sum(cfg.pages(b) for b in range(cfg.B)) * cfg.H_kv),
            "ncu dram__bytes_read+write of the 2^18-token case scaled by rows"),
        "e2e": {"value": round(e2e_us, 2), "unit": "us/step", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": N_LAUNCH * K,
        "clocks": clk,
    }
    # the dominant kernel (the largest share of the step's kernel time): the
    # fused attention, on the bytes it must read (keys of the selected
    # page-heads, values of those holding weight)
    one_m = cfg.B == 1 and cfg.lengths[0] == 1 << 20
    line["roofline"] = roofline_entry(
        "entmax_bf16_kernel (entmaxkv_sparse_attend: K pass, threshold, V pass)", by["attend"], attend_us, peak,
        ATTEND_DRAM_BYTES_1M if one_m else None,
        "algorithmic bytes: keys of the selected page-heads plus values of those holding weight (mean over the "
        "timed steps); traffic: ncu dram__bytes_read+write of one launch of this workload")
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


# ---------------------------------------------------------------- native arm
def timed_replays(gs, step, toks, warm, steps, flush, stream, stages=False):
    """`warm` + `steps` replays of a graphed step, issued back to back with no
    host synchronisation: per step the step's inputs are copied in (device to
    device), the L2 is flushed (L2Flush) and the replay is bracketed by
    CUDA events on the stream; the selected and loaded-value page counts add up
    on the device.  Returns (per-step us, mean selected page-heads, mean value
    page-heads, mean stage us or None)."""
    sel_acc = torch.zeros((), dtype=torch.int64, device="cuda")
    vp_acc = torch.zeros((), dtype=torch.int64, device="cuda")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    stage_sum = None
    for i in range(warm + steps):
        k, v, q = toks[i]
        gs.q.copy_(q)
        gs.k.copy_(k)
        gs.v.copy_(v)
        step.v_pages.zero_()
        flush(i)
        j = i - warm
        if j >= 0:
            ev[j][0].record(stream)
        gs.replay()
        if j >= 0:
            ev[j][1].record(stream)
            sel_acc += step.sel_count.sum()
            vp_acc += step.v_pages.sum()
            if stages:   # event nodes of the instrumented graph: read after each replay
                torch.cuda.synchronize()
                st = gs.stage_us()
                stage_sum = dict(st) if stage_sum is None else {n: stage_sum[n] + st[n] for n in st}
    torch.cuda.synchronize()
    step.check()
    us = [a.elapsed_time(b) * 1e3 for a, b in ev]
    stage = {n: x / steps for n, x in stage_sum.items()} if stage_sum else None
    return us, sel_acc.item() / steps, vp_acc.item() / steps, stage


def decode_tokens(wl, first, n):
    return [wl.decode_token(first + i) for i in range(n)]


def run_native(args, rank, world, local):
    from sparse_long_context_min_b200.step import DecodeStep, GraphedStep, build_pool

    torch.manual_seed(0)
    K, W = args.steps, args.warmup
    Ks = min(K, 200)                         # replays of the instrumented graph (stage breakdown)
    Kg = min(K, 200)                         # Gaussian-selector replays
    # tokens appended during the run: the top-k graphs, the e2e leg, the Gaussian graph
    appends = (W + K) + (W + Ks) + (W + K) + (W + Kg) + 64
    wl = make_workload(args.context, rank, appends=appends)
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    flush = L2Flush()

    # ---- headline: top-k 1/64, K graphed steps bracketed by barrier + sync
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 64, alpha=cfg.alpha)
    plain = GraphedStep(step, append=True, stage_events=False)
    inst = GraphedStep(step, append=True, stage_events=True)
    toks = decode_tokens(wl, 0, W + K)
    clocks = Clocks(local, interval_ms=10)
    barrier(world)
    torch.cuda.synchronize()
    with clocks:
        step_us, sel_total, v_total, _ = timed_replays(plain, step, toks, W, K, flush, stream)
    torch.cuda.synchronize()
    barrier(world)
    mean_us = statistics.mean(step_us)
    mean_us_all = max_over_ranks(mean_us, world)
    best_us_all = max_over_ranks(min(step_us), world)
    median_us_all = max_over_ranks(statistics.median(step_us), world)
    del toks
    # stage breakdown from the instrumented graph (outside the timed region)
    toks = decode_tokens(wl, W + K, W + Ks)
    _, _, _, stage = timed_replays(inst, step, toks, W, Ks, flush, stream, stages=True)
    del toks
    score_us = max_over_ranks(stage["score"], world)
    attend_us = max_over_ranks(stage["attend"], world)

    # ---- e2e through the C ABI with host buffers (copies inside the timed region)
    e2e_us, h2d, d2h = run_e2e(wl, pool, seq_lens, K, W, flush)
    e2e_us = max_over_ranks(e2e_us, world)

    extra = {}
    if not args.no_baselines:
        gstep = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "gauss", alpha=cfg.alpha, delta=0.5)
        ggraph = GraphedStep(gstep, append=True, stage_events=False)
        toks = decode_tokens(wl, 3 * (W + K), W + Kg)
        g_us, g_sel, g_v, _ = timed_replays(ggraph, gstep, toks, W, Kg, flush, stream)
        del toks, ggraph
        extra["gauss_value_pages"] = round(g_v, 1)
        extra["gauss_us_per_step"] = round(max_over_ranks(statistics.mean(g_us), world), 2)
        extra["gauss_selected_pages"] = round(g_sel, 1)
        fe, fs = run_full(wl, pool, seq_lens, flush)
        fe, fs = max_over_ranks(fe, world), max_over_ranks(fs, world)
        extra["full_entmax_us"] = round(fe, 1)
        extra["full_softmax_us"] = round(fs, 1)
        extra["topk_speedup_vs_full_entmax"] = round(fe / mean_us_all, 2)
        extra["topk_speedup_vs_full_softmax"] = round(fs / mean_us_all, 2)
        extra["gauss_speedup_vs_full_entmax"] = round(fe / extra["gauss_us_per_step"], 2)
        extra["gauss_speedup_vs_full_softmax"] = round(fs / extra["gauss_us_per_step"], 2)
        extra.update({k: round(max_over_ranks(v, world), 2)
                      for k, v in run_attend_variants(wl, pool, seq_lens, flush).items()})
        extra["attend_variants_note"] = ("eager calls between events on one top-k 1/64 selection; "
                                         "include launch latency not hidden by a graph")
    del pool
    torch.cuda.empty_cache()
    if world == 1 and not args.no_configs:
        extra["per_config"] = config_legs(flush, W, min(K, 200), hbm_peak())

    cpu = None
    if rank == 0 and not args.no_cpu:
        cpu = cpu_baseline_subprocess(args.context, args.leg_seconds)

    line = native_line(cfg, world, K, W, mean_us_all, best_us_all, median_us_all, score_us, stage, sel_total,
                       v_total, extra, (e2e_us, h2d, d2h), clocks.summary(), cpu, hbm_peak(), attend_us)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(wl, pool, seq_lens, K, W, flush):
    """Same step through the public API (the graphed step) with the step's
    inputs in pinned host memory: one H2D copy of q and the new token (packed
    by GraphedStep.pack_host); the result is written by the attention kernel
    straight into pinned host memory (the D2H transfer of the output) inside
    the events."""
    from sparse_long_context_min_b200.step import DecodeStep, GraphedStep
    cfg = wl.cfg
    stream = torch.cuda.current_stream()
    out_h = torch.empty(cfg.B, cfg.H_q, cfg.d, dtype=torch.float32).pin_memory()
    st = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 64, alpha=cfg.alpha,
                    out=out_h)
    gs = GraphedStep(st, append=True, stage_events=False)
    host = []
    for i in range(W + K):
        k, v, q = wl.decode_token(1_000_000 + i)
        host.append(gs.pack_host(k, v, q))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(W + K):
        flush(i)
        j = i - W
        if j >= 0:
            ev[j][0].record(stream)
        gs.inputs.copy_(host[i], non_blocking=True)
        gs.replay()
        if j >= 0:
            ev[j][1].record(stream)
    torch.cuda.synchronize()
    st.check()
    us = statistics.mean(a.elapsed_time(b) * 1e3 for a, b in ev)
    h2d = host[0].numel() * host[0].element_size()
    d2h = out_h.numel() * out_h.element_size()
    return us, h2d, d2h


def run_full(wl, pool, seq_lens, flush, reps=5, warm=3):
    """Full-cache entmax and softmax decode over every page (the baselines)."""
    from sparse_long_context_min_b200 import binding as BND
    cfg = wl.cfg
    stream = torch.cuda.current_stream()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(cfg.B, cfg.H_q, cfg.d, device="cuda")
    res = []
    for op in (BND.OP_FULL_ENTMAX, BND.OP_FULL_SOFTMAX):
        ws = torch.empty(BND.workspace_size(op, cfg.B, cfg.H_q, cfg.H_kv, wl.max_pages, 0, cfg.ps, cfg.d),
                         dtype=torch.uint8, device="cuda")
        times = []
        for i in range(warm + reps):
            flush(i)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            if op == BND.OP_FULL_ENTMAX:
                BND.full_entmax_decode(pool, wl.q, wl.page_table, seq_lens, cfg.alpha, cfg.scale, out, ws, st)
            else:
                BND.full_softmax_decode(pool, wl.q, wl.page_table, seq_lens, cfg.scale, out, ws, st)
            b.record(stream)
            if i >= warm:
                times.append((a, b))
        torch.cuda.synchronize()
        if int(st.item()):
            raise BND.EntmaxKVError(int(st.item()), "full-cache baseline")
        res.append(statistics.mean(a.elapsed_time(b) * 1e3 for a, b in times))
        del ws
    return res[0], res[1]


def run_attend_variants(wl, pool, seq_lens, flush, reps=5, warm=3):
    """On one top-k 1/64 selection: sparse entmax attention (alpha 1.5, the
    step's), softmax over the same pages (the matched-budget baseline) and
    entmax with alpha = 1.25 (no closed form: Newton threshold, powf weights);
    and the Gaussian selection with alpha = 3 (quadrature expectations)."""
    from sparse_long_context_min_b200 import binding as BND
    from sparse_long_context_min_b200.step import DecodeStep
    cfg = wl.cfg
    stream = torch.cuda.current_stream()
    step = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "topk", budget_frac=1 / 64, alpha=cfg.alpha)
    step.score(wl.q)
    step.choose()
    out = torch.empty_like(step.out)
    ws_s = torch.empty(BND.workspace_size(BND.OP_SPARSE_SOFTMAX, cfg.B, cfg.H_q, cfg.H_kv, wl.max_pages,
                                          step.k_max, cfg.ps, cfg.d), dtype=torch.uint8, device="cuda")
    calls = {
        "sparse_entmax_attend_us": lambda: BND.sparse_attend(pool, wl.q, wl.page_table, seq_lens, step.sel,
                                                             step.sel_count, cfg.alpha, cfg.scale, out,
                                                             step.workspace, step.status),
        "matched_budget_sparse_softmax_attend_us": lambda: BND.sparse_softmax_attend(
            pool, wl.q, wl.page_table, seq_lens, step.sel, step.sel_count, cfg.scale, out, ws_s, step.status),
        "sparse_entmax_alpha_1.25_attend_us": lambda: BND.sparse_attend(pool, wl.q, wl.page_table, seq_lens,
                                                                        step.sel, step.sel_count, 1.25, cfg.scale,
                                                                        out, step.workspace, step.status),
    }
    gstep = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, "gauss", alpha=3.0, delta=0.5)
    gstep.score(wl.q)
    calls["gauss_select_alpha_3_us"] = gstep.choose     # quadrature expectations (no closed form)
    res = {}
    for name, fn in calls.items():
        times = []
        for i in range(warm + reps):
            flush(i)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            if i >= warm:
                times.append((a, b))
        torch.cuda.synchronize()
        res[name] = round(statistics.mean(a.elapsed_time(b) * 1e3 for a, b in times), 2)
    step.check()
    gstep.check()
    return res


def config_legs(flush, W, steps, peak):
    """One-GPU timings of the other benchmark configurations at their stated
    sizes, each step graphed with its token append and the L2 flushed between
    steps: configuration 2 (131072 tokens, top-k budgets of 64, 128 and 256
    pages), 3 (B = 4 x 262144 tokens, Gaussian selector, alpha in {1.5, 2},
    Delta in {0, 0.5, 1}) and 5 (ragged B = 1, 8, 32, top-k 1/16).  Per leg:
    us per step, algorithmic bytes, GB/s and the fraction of the copy peak."""
    import dataclasses
    from sparse_long_context_min_b200 import workloads
    from sparse_long_context_min_b200.step import DecodeStep, GraphedStep, build_pool
    stream = torch.cuda.current_stream()
    peak_gbs = peak[0]
    out = {}

    def leg(wl, pool, seq_lens, name, mode, first, **kw):
        cfg = wl.cfg
        st = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, mode, alpha=kw.pop("alpha", cfg.alpha), **kw)
        gs = GraphedStep(st, append=True, stage_events=False)
        toks = decode_tokens(wl, first, W + steps)
        us, sel, vp, _ = timed_replays(gs, st, toks, W, steps, flush, stream)
        mean = statistics.mean(us)
        by = algorithmic_bytes(cfg, sel, vp, mode)["total"]
        gbs = by / (mean * 1e-6) / 1e9
        out[name] = {"us_per_step": round(mean, 2), "selected_page_heads": round(sel, 1),
                     "value_page_heads": round(vp, 1), "algorithmic_bytes": int(by), "gbs": round(gbs, 1),
                     "frac_of_measured_hbm": round(gbs / peak_gbs, 4), "frac_of_8tbs": round(gbs / HBM_NOMINAL_GBS, 4)}
        del gs, st, toks

    per = W + steps
    c2 = workloads.config(2)
    wl = workloads.Workload(dataclasses.replace(c2, decode_steps=3 * per + 64), device="cuda")
    pool, lens = build_pool(wl)
    for i, budget in enumerate(c2.budgets):
        leg(wl, pool, lens, "config2_topk_%d_pages" % budget, "topk", i * per, budget=budget)
    del wl, pool, lens
    torch.cuda.empty_cache()
    c3 = workloads.config(3)
    wl = workloads.Workload(dataclasses.replace(c3, decode_steps=6 * per + 64), device="cuda")
    pool, lens = build_pool(wl)
    i = 0
    for alpha in c3.alphas:
        for delta in c3.deltas:
            leg(wl, pool, lens, "config3_gauss_alpha%g_delta%g" % (alpha, delta), "gauss", i * per, alpha=alpha,
                delta=delta)
            i += 1
    del wl, pool, lens
    torch.cuda.empty_cache()
    for B in (1, 8, 32):
        c5 = workloads.config(5, B=B)
        wl = workloads.Workload(dataclasses.replace(c5, decode_steps=per + 64), device="cuda")
        pool, lens = build_pool(wl)
        leg(wl, pool, lens, "config5_ragged_B%d_topk_1_16" % B, "topk", 0, budget_frac=c5.budget_frac)
        del wl, pool, lens
        torch.cuda.empty_cache()
    out["note"] = ("graphed steps with the token append, L2 flushed between steps, %d timed after %d warm-up; "
                   "bytes counted as for the headline (metadata of every page, keys of the kept page-heads, values "
                   "of those holding weight, append, page table, output)" % (steps, W))
    return out


# ---------------------------------------------------------------- oracle timing
# The oracle runs in a process that never touches the GPU: its data are
# generated on the host, then a pool of worker processes forked from it shares
# them (copy on write) to time the all-core leg.
_LEG = {}


def _widen(u16):
    """bf16 bit patterns (uint16 / int16 numpy) -> float32, exactly."""
    import numpy as np
    return (u16.astype(np.uint32) << 16).view(np.float32)


def _leg_setup(context):
    import numpy as np
    from oracle import replica
    wl = make_workload(context, 0, device="cpu")
    cfg = wl.cfg
    keys, vals = wl.sequence(0)
    kb = keys.view(torch.int16).numpy().view(np.uint16)
    vb = vals.view(torch.int16).numpy().view(np.uint16)
    # the page metadata exists before a decode step: built once, outside the timing
    metas = [replica.page_meta(_widen(kb[g]), cfg.ps) for g in range(cfg.H_kv)]
    _LEG.update(cfg=cfg, q=wl.q[0].numpy(), k=kb, v=vb, metas=metas,
                scale32=float(np.float32(1.0 / math.sqrt(cfg.d))))


def _leg_sparse_head(g):
    """The oracle's sparse step for kv head g: replica bounds over every page,
    top-k 1/64, float64 entmax attention over the kept pages."""
    from oracle import attend, replica, select
    cfg = _LEG["cfg"]
    G = cfg.G
    qg = _LEG["q"][g * G:(g + 1) * G]
    m = _LEG["metas"][g]
    _, ubg = replica.bound(qg, m["kmin"], m["kmax"], _LEG["scale32"])
    pages = select.topk(ubg, select.budget_pages(len(ubg), -1, 1 / 64))
    tok = attend.token_indices(pages, cfg.lengths[0], cfg.ps)
    o, _, _ = attend.entmax_attention(qg, _widen(_LEG["k"][g][tok]), _widen(_LEG["v"][g][tok]), cfg.alpha,
                                      1.0 / math.sqrt(cfg.d))
    return float(o[0, 0])


def _leg_full_head(g):
    """The oracle's full-cache entmax decode for kv head g (every token)."""
    from oracle import attend
    cfg = _LEG["cfg"]
    G = cfg.G
    o, _, _ = attend.entmax_attention(_LEG["q"][g * G:(g + 1) * G], _widen(_LEG["k"][g]), _widen(_LEG["v"][g]),
                                      cfg.alpha, 1.0 / math.sqrt(cfg.d))
    return float(o[0, 0])


def _leg_cores():
    return len(os.sched_getaffinity(0))


def _leg_pool(n):
    import multiprocessing as mp
    return mp.get_context("fork").Pool(n)


def oracle_leg(context, seconds):
    """The oracle, as it stands, timed on this host's cores (this process must
    not have touched the GPU): a sparse decode step over the 8 kv heads on one
    core and on min(cores, 8) worker processes (one kv head each), and the
    full-cache entmax decode of one kv head on one core, scaled to the 8."""
    _leg_setup(context)
    cfg = _LEG["cfg"]
    H = cfg.H_kv
    t0 = time.perf_counter()
    n1 = 0
    while True:
        for g in range(H):
            _leg_sparse_head(g)
        n1 += 1
        if time.perf_counter() - t0 > seconds:
            break
    single = (time.perf_counter() - t0) / n1
    cores = _leg_cores()
    workers = max(1, min(cores, H))
    with _leg_pool(workers) as pool:
        pool.map(_leg_sparse_head, range(H))                   # start-up and warm
        t0 = time.perf_counter()
        nm = 0
        while True:
            pool.map(_leg_sparse_head, range(H))
            nm += 1
            if time.perf_counter() - t0 > seconds:
                break
        multi = (time.perf_counter() - t0) / nm
    t0 = time.perf_counter()
    _leg_full_head(0)
    full = (time.perf_counter() - t0) * H
    return {"value": round(multi * 1e6, 1), "unit": "us/step", "cores": workers, "kind": "oracle",
            "host_cores": cores, "single_core_us_per_step": round(single * 1e6, 1),
            "full_cache_us_per_step_single_core": round(full * 1e6, 1),
            "sample": ("the sparse decode step of the bench workload (%d tokens): replica bounds over every page, "
                       "top-k 1/64, float64 entmax attention over the kept pages, for each of the 8 kv heads; "
                       "value = %d worker processes, one kv head each, %d steps; single core %d steps; full-cache "
                       "entmax decode of kv head 0 on one core, scaled x8" % (context, workers, nm, n1))}


def cpu_baseline_subprocess(context, seconds):
    """oracle_leg in a fresh process (this one holds a CUDA context, and the
    oracle's worker pool is forked)."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--oracle-leg", "--context", str(context),
                        "--leg-seconds", str(seconds)], capture_output=True, text=True, timeout=1800,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    if r.returncode != 0 or not lines:
        raise RuntimeError("oracle leg failed: " + r.stderr[-2000:])
    return json.loads(lines[-1])


def run_reference(args, rank, world):
    """The reference arm: the oracle, as it stands, on this host's cores (no
    GPU); each step is the sparse decode step over the 8 kv heads on
    min(cores, 8) worker processes, one kv head each."""
    if rank != 0:
        return
    _leg_setup(args.context)
    cfg = _LEG["cfg"]
    H = cfg.H_kv
    workers = max(1, min(_leg_cores(), H))
    with _leg_pool(workers) as pool:
        for _ in range(args.warmup):
            pool.map(_leg_sparse_head, range(H))
        t0 = time.perf_counter()
        for _ in range(args.steps):
            pool.map(_leg_sparse_head, range(H))
        per = (time.perf_counter() - t0) / args.steps * 1e6
    sample = ("sparse decode step over the 8 kv heads (replica bounds over every page, top-k 1/64, float64 entmax "
              "attention over the kept pages; page metadata built before timing, no token appended), %d worker "
              "processes, one kv head each" % workers)
    line = {"metric": METRIC, "value": round(per, 1), "unit": "us/step", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(per / 1e3, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(cfg.lengths[0]),
                       "seq_len": cfg.lengths[0]},
            "impl": "reference",
            "cpu_baseline": {"value": round(per, 1), "unit": "us/step", "cores": workers, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(per, 1), "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def selector_sweep(args):
    """The two selectors against context length on configuration 4's generator
    (B = 1, 32/8 heads, d = 128, pages of 64, bf16): us per graphed step with
    its token append, selected and loaded-value page-heads, algorithmic bytes
    and GB/s, for top-k 1/64 and the Gaussian selector with Delta = 0.5."""
    from sparse_long_context_min_b200.step import DecodeStep, GraphedStep, build_pool
    torch.cuda.set_device(0)
    W, K = args.warmup, min(args.steps, 200)
    stream = torch.cuda.current_stream()
    flush = L2Flush()
    for ctx in (1 << 18, 1 << 19, 1 << 20):
        wl = make_workload(ctx, 0, appends=2 * (W + K) + 64)
        cfg = wl.cfg
        pool, lens = build_pool(wl)
        for i, mode in enumerate(("topk", "gauss")):
            st = DecodeStep(pool, wl.page_table, lens, cfg.H_q, mode, budget_frac=1 / 64, alpha=cfg.alpha,
                            delta=0.5)
            gs = GraphedStep(st, append=True, stage_events=False)
            toks = decode_tokens(wl, i * (W + K), W + K)
            us, sel, vp, _ = timed_replays(gs, st, toks, W, K, flush, stream)
            mean = statistics.mean(us)
            by = algorithmic_bytes(cfg, sel, vp, mode)["total"]
            print(json.dumps({"context": ctx, "selector": "top-k 1/64" if mode == "topk" else "gaussian delta 0.5",
                              "us_per_step": round(mean, 2), "selected_page_heads": round(sel, 1),
                              "value_page_heads": round(vp, 1), "pages_per_kv_head": cfg.pages(0),
                              "algorithmic_bytes": int(by), "gbs": round(by / (mean * 1e-6) / 1e9, 1)}), flush=True)
            del gs, st, toks
        del pool, lens, wl
        torch.cuda.empty_cache()


def replay_only(args):
    """Capture one decode step (top-k 1/64 or the Gaussian selector, Delta 0.5)
    of the bench workload as a graph and replay it; prints nothing but "ok"."""
    from sparse_long_context_min_b200.step import DecodeStep, GraphedStep, build_pool
    wl = make_workload(args.context, 0)
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    st = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, args.replay_only, budget_frac=1 / 64,
                    alpha=cfg.alpha, delta=0.5)
    gs = GraphedStep(st, append=True, stage_events=False)
    flush = L2Flush()
    for i in range(args.steps):
        k, v, q = wl.decode_token(i)
        gs.inputs.copy_(gs.pack_host(k, v, q), non_blocking=True)
        flush(i)
        gs.replay()
    torch.cuda.synchronize()
    st.check()
    print("ok", args.replay_only)


def main():
    args = parse()
    if args.oracle_leg:
        print(json.dumps(oracle_leg(args.context, args.leg_seconds)), flush=True)
        return
    if args.replay_only:
        torch.cuda.set_device(0)
        replay_only(args)
        return
    if args.selector_sweep:
        selector_sweep(args)
        return
    rank, world, local = dist_init(args.gpus, "gloo" if args.impl == "reference" else "nccl")
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_native(args, rank, world, local)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
