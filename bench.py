"""Benchmark: one EntmaxKV decode step at 1M-token context on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

A step is the whole decode path on one batch: append the step's token (KV
write + page metadata), score every page (bounding-box bound), select the top
1/64 of pages per kv head, and run exact 1.5-entmax attention over the
selected pages.  Workload: B=1 sequence of 2^20 tokens per GPU, 32 query / 8
kv heads, head dim 128, pages of 64, bf16 cache (synthetic clustered keys with
planted tokens).  L2 is flushed (a 256 MiB write) between timed steps, outside
the per-step CUDA events.  Rank 0 prints one JSON line.

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
# capture of the 2^18-token case (16,842,240 bytes for 4097 pages x 8 heads);
# scaled by rows to the bench launch.  Must be re-measured when the scoring
# kernel changes.
SCORE_DRAM_BYTES_PER_ROW = 16842240 / (4097 * 8)
HBM_NOMINAL_GBS = 8000.0
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
MiB = 1 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--context", type=int, default=1 << 20, help="tokens per sequence (default 2^20)")
    ap.add_argument("--no-baselines", action="store_true", help="skip the full-cache and Gaussian timings")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline leg")
    ap.add_argument("--replay-only", choices=["topk", "gauss"], default=None,
                    help="build the workload, capture that step as a graph and replay it --steps times "
                         "without timing (a short program for profiler launch lists)")
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


N_LAUNCH = 6   # per step: append (one token, no separate length kernel), score, top-k, qk, tau, pv


def native_line(cfg, world, K, W, mean_us, best_us, median_us, score_us, stage, sel_total, v_total, extra, e2e,
                clk, cpu, peak):
    """The native arm's JSON line from the measured numbers (times are the
    max over ranks; e2e = (us per step, H2D bytes, D2H bytes); peak = (GB/s,
    "measured" or "fallback"))."""
    by = algorithmic_bytes(cfg, sel_total, v_total, "topk")
    peak_gbs, peak_kind = peak
    e2e_us, h2d, d2h = e2e
    step_gbs = by["total"] / (mean_us * 1e-6) / 1e9
    score_gbs = by["score"] / (score_us * 1e-6) / 1e9
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
            "l2": "flushed between steps (256 MiB write outside the step events)",
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
        "roofline": {
            "kernel": "score_box16_kernel (entmaxkv_score_pages, bbox, bf16)",
            "bound": "hbm",
            "achieved": round(score_gbs, 1),
            "peak": peak_gbs,
            "peak_kind": peak_kind,
            "unit": "GB/s",
            "frac": round(score_gbs / peak_gbs, 4),
            "traffic": round(SCORE_DRAM_BYTES_PER_ROW * sum(cfg.pages(b) for b in range(cfg.B)) * cfg.H_kv),
            "traffic_note": "ncu dram__bytes_read+write of the 2^18-token case scaled by rows",
            "bytes_per_launch": by["score"],
        },
        "e2e": {"value": round(e2e_us, 2), "unit": "us/step", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": N_LAUNCH * K,
        "clocks": clk,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


# ---------------------------------------------------------------- native arm
def run_native(args, rank, world, local):
    import numpy as np
    from sparse_long_context_min_b200 import binding as BND
    from sparse_long_context_min_b200.step import DecodeStep, GraphedStep, build_pool

    torch.manual_seed(0)
    # tokens appended during the run: top-k (two graphs) + e2e + Gaussian (two graphs)
    appends = 3 * (args.steps + args.warmup) + 2 * (max(3, args.steps // 4) + 3) + 64
    wl = make_workload(args.context, rank, appends=appends)
    cfg = wl.cfg
    pool, seq_lens = build_pool(wl)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * MiB, dtype=torch.uint8, device="cuda")
    K, W = args.steps, args.warmup
    total_steps = W + K

    def one_mode(mode, budget_frac=1 / 64, delta=0.5, steps=None, warm=None):
        """K graphed steps timed with events around each replay (plain graph, so
        kernels overlap across stage boundaries), then K replays of a graph with
        event nodes between stages for the per-stage breakdown.  Returns per-step
        us, mean stage us, mean selected and loaded-value page-heads per step."""
        steps = K if steps is None else steps
        warm = W if warm is None else warm
        st = DecodeStep(pool, wl.page_table, seq_lens, cfg.H_q, mode, budget_frac=budget_frac, alpha=cfg.alpha,
                        delta=delta)
        plain = GraphedStep(st, append=True, stage_events=False)
        inst = GraphedStep(st, append=True, stage_events=True)
        toks = [wl.decode_token(i) for i in range(2 * (warm + steps))]
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        step_us, stages, sel, vp = [], [], [], []
        for phase, gs in (("step", plain), ("stages", inst)):
            for i in range(warm + steps):
                k, v, q = toks[(0 if phase == "step" else warm + steps) + i]
                gs.q.copy_(q)
                gs.k.copy_(k)
                gs.v.copy_(v)
                st.v_pages.zero_()
                flush.fill_(i & 0xFF)
                e0.record(stream)
                gs.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                if i < warm:
                    continue
                if phase == "step":
                    step_us.append(e0.elapsed_time(e1) * 1e3)
                    sel.append(int(st.sel_count.sum().item()))
                    vp.append(int(st.v_pages.sum().item()))
                else:
                    stages.append(gs.stage_us())
        st.check()
        stage = {n: statistics.mean(x[n] for x in stages) for n in GraphedStep.STAGES} if stages[0] else {}
        return step_us, stage, statistics.mean(sel), statistics.mean(vp)

    # ---- headline: top-k 1/64, timed K steps bracketed by barrier + sync
    clocks = Clocks(local)
    barrier(world)
    torch.cuda.synchronize()
    with clocks:
        step_us, stage, sel_total, v_total = one_mode("topk")
    torch.cuda.synchronize()
    barrier(world)
    mean_us = statistics.mean(step_us)
    mean_us_all = max_over_ranks(mean_us, world)
    best_us_all = max_over_ranks(min(step_us), world)
    median_us_all = max_over_ranks(statistics.median(step_us), world)
    score_us = max_over_ranks(stage["score"], world)

    # ---- e2e through the C ABI with host buffers (copies inside the timed region)
    e2e_us, h2d, d2h = run_e2e(wl, pool, seq_lens, K, W, flush)
    e2e_us = max_over_ranks(e2e_us, world)

    extra = {}
    if not args.no_baselines:
        g_us, g_stage, g_sel, g_v = one_mode("gauss", steps=max(3, K // 4), warm=3)
        extra["gauss_value_pages"] = round(g_v, 1)
        extra["gauss_us_per_step"] = round(max_over_ranks(statistics.mean(g_us), world), 2)
        extra["gauss_selected_pages"] = round(g_sel, 1)
        extra["gauss_stage_us"] = {k: round(v, 2) for k, v in g_stage.items()}
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

    cpu = None
    if rank == 0 and not args.no_cpu:
        cpu = cpu_baseline(wl, pool, budget_frac=1 / 64, seconds=8.0)

    line = native_line(cfg, world, K, W, mean_us_all, best_us_all, median_us_all, score_us, stage, sel_total,
                       v_total, extra, (e2e_us, h2d, d2h), clocks.summary(), cpu, hbm_peak())
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(wl, pool, seq_lens, K, W, flush):
    """Same step through the public API (the graphed step) with the step's
    inputs in pinned host memory: one H2D copy of q and the new token (packed
    by GraphedStep.pack_host); the result is written by the attention kernels
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
        k, v, q = wl.decode_token(10_000 + i)
        host.append(gs.pack_host(k, v, q))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(W + K):
        flush.fill_(i & 0xFF)
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
            flush.fill_(i & 0xFF)
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
            flush.fill_(i & 0xFF)
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


# ---------------------------------------------------------------- oracle timing
def oracle_sample(wl, g, budget_frac, meta, keys, vals):
    """The oracle's sparse step for kv head g: replica bounds, top-k, entmax attention."""
    from oracle import attend, replica, select
    cfg = wl.cfg
    qg = wl.q[0, g * cfg.G:(g + 1) * cfg.G].cpu().numpy()
    _, ubg = replica.bound(qg, meta["kmin"], meta["kmax"], float(torch.tensor(cfg.scale, dtype=torch.float32)))
    pages = select.topk(ubg, select.budget_pages(len(ubg), -1, budget_frac))
    tok = attend.token_indices(pages, cfg.lengths[0], cfg.ps)
    o, tau, _ = attend.entmax_attention(qg, keys[tok], vals[tok], cfg.alpha, 1.0 / math.sqrt(cfg.d))
    return o


def cpu_baseline(wl, pool, budget_frac, seconds):
    """Time the oracle (as it stands) on the host cores: one kv head's share of
    the sparse step, repeated for about `seconds`, scaled to the 8 heads."""
    from oracle import replica
    cfg = wl.cfg
    keys, vals = wl.sequence(0, heads=[0])
    keys = keys[0].float().cpu().numpy()
    vals = vals[0].float().cpu().numpy()
    meta = replica.page_meta(keys, cfg.ps)          # metadata exists before a decode step
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_sample(wl, 0, budget_frac, meta, keys, vals)
        n += 1
        if time.perf_counter() - t0 > seconds:
            break
    per_head = (time.perf_counter() - t0) / n
    us = per_head * cfg.H_kv * 1e6
    return {"value": round(us, 1), "unit": "us/step", "cores": 1, "kind": "oracle",
            "sample": "kv head 0 of 8 (4 query heads): replica bounds over all 16384 pages, top-k, float64 "
                      "entmax attention over the 256 kept pages; %d repetitions, scaled x8 to a full step" % n}


def run_reference(args, rank, world):
    if rank != 0:
        return
    if torch.cuda.is_available():
        torch.cuda.set_device(0)
    wl = make_workload(args.context, 0, device="cuda" if torch.cuda.is_available() else "cpu")
    from oracle import replica
    cfg = wl.cfg
    keys, vals = wl.sequence(0, heads=[0])
    keys = keys[0].float().cpu().numpy()
    vals = vals[0].float().cpu().numpy()
    meta = replica.page_meta(keys, cfg.ps)
    for _ in range(args.warmup):
        oracle_sample(wl, 0, 1 / 64, meta, keys, vals)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(wl, 0, 1 / 64, meta, keys, vals)
    per = (time.perf_counter() - t0) / args.steps * cfg.H_kv * 1e6
    sample = ("kv head 0 of 8 per step (replica bounds over all pages, top-k, float64 entmax attention over "
              "the kept pages; page metadata built before timing, no token appended), scaled x8")
    line = {"metric": METRIC, "value": round(per, 1), "unit": "us/step", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(per / 1e3, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(cfg.lengths[0]),
                       "seq_len": cfg.lengths[0]},
            "impl": "reference",
            "cpu_baseline": {"value": round(per, 1), "unit": "us/step", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(per, 1), "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


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
    flush = torch.empty(256 * MiB, dtype=torch.uint8, device="cuda")
    for i in range(args.steps):
        k, v, q = wl.decode_token(i)
        gs.inputs.copy_(gs.pack_host(k, v, q), non_blocking=True)
        flush.fill_(i & 0xFF)
        gs.replay()
    torch.cuda.synchronize()
    st.check()
    print("ok", args.replay_only)


def main():
    args = parse()
    if args.replay_only:
        torch.cuda.set_device(0)
        replay_only(args)
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
