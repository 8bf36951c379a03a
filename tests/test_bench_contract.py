"""bench.py's host side on the CPU: the reference arm's JSON line (alone and
under torchrun with two gloo ranks, where rank 0 alone prints), the workload
name both arms share, and the algorithmic byte count of a step against a
count by hand."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _check_reference_line(line, n):
    d = json.loads(line)
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["n_gpus"] == n and d["higher_is_better"] is False
    assert d["metric"] == bench.METRIC and d["unit"] == "us/step" and d["value"] > 0
    assert d["config"]["workload"] == bench.workload_name(65536)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and 1 <= cb["cores"] <= 8 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


ARGS = ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1", "--context", "65536"]


def test_reference_arm_one_process():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable] + ARGS, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    _check_reference_line(lines[0], 1)


def test_reference_arm_two_ranks_rank0_prints_once():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_port())] + ARGS + ["--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    _check_reference_line(lines[0], 2)


def test_workload_names():
    assert bench.workload_name(1 << 20).startswith("million-token decode: B=1 x 1048576 tokens per GPU")
    assert bench.workload_name(65536).startswith("decode at 65536 tokens: B=1 x 65536 tokens")


def test_algorithmic_bytes_by_hand():
    """The million-token step after one appended token: 16385 pages per kv head,
    257 pages kept per kv head (2056 page-heads), 278 of them holding weight."""
    import dataclasses
    from sparse_long_context_min_b200 import workloads
    cfg = dataclasses.replace(workloads.config(4), lengths=[(1 << 20) + 1])
    by = bench.algorithmic_bytes(cfg, 2056, 278, "topk")
    P = 16385
    kmin_kmax = P * 8 * 128 * 2 * 2              # bf16 k_min and k_max of every (page, kv head)
    bounds = 8 * P * 4                           # fp32 bound per (kv head, page), written
    table = P * 4
    keys = 2056 * 64 * 128 * 2                   # K of the kept page-heads
    values = 278 * 64 * 128 * 2                  # V of the page-heads holding weight
    append = 8 * 128 * 2 * 2 + 8 * 128 * 2 * (2 * 2 + 2 * 4)   # token K, V; metadata row read + write
    out = 32 * 128 * 4
    assert by["score"] == kmin_kmax + bounds + table
    assert by["attend"] == keys + values
    assert by["total"] == kmin_kmax + bounds + table + keys + values + append + out
    assert abs(by["total"] / 1e6 - 105.99) < 0.01
    g = bench.algorithmic_bytes(cfg, 0, 0, "gauss")
    assert g["score"] == P * 8 * 128 * 2 * 4 + 3 * 32 * P * 4 + table    # mean, m2 read; m, v, est written


FAKE_SMI = r'''#!{python}
"""Stand-in for nvidia-smi: answers the one-shot index query, and in loop
mode prints one CSV sample per interval until SIGINT."""
import datetime, signal, sys, time
args = sys.argv[1:]
target = args[args.index("-i") + 1]
if target not in ("0", "0000ABCD:3B:00.0"):
    sys.exit(6)
if "--query-gpu=index" in args:
    print("0")
    sys.exit(0)
ms = int(args[args.index("-lms") + 1])
stop = []
signal.signal(signal.SIGINT, lambda *a: stop.append(1))
i = 0
while not stop:
    ts = datetime.datetime.now().strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    slow = "Active" if {slow_from} <= i else "Not Active"
    print("%s, 0, %d, 1965, 700.0, 0x0, %s, Not Active, Not Active, Not Active" % (ts, 1965 - i, slow), flush=True)
    i += 1
    time.sleep(ms / 1000.0)
'''


def _fake_smi(tmp_path, slow_from=10 ** 9):
    p = tmp_path / "nvidia-smi"
    p.write_text(FAKE_SMI.replace("{python}", sys.executable).replace("{slow_from}", str(slow_from)))
    p.chmod(0o755)
    return str(p)


def test_clock_sampler_keeps_the_timed_region(tmp_path):
    import datetime
    import statistics
    import time
    c = bench.Clocks(0, interval_ms=20, lead_s=0.6, smi=_fake_smi(tmp_path))
    with c:
        time.sleep(0.3)
    s = c.summary()
    stamp = lambda l: datetime.datetime.strptime(l.split(",")[0], bench.Clocks.TS_FORMAT)  # noqa: E731
    inside = [l for l in c.lines if c.t0 <= stamp(l) <= c.t1]
    assert s["window"] == "timed region" and s["samples"] == len(inside) >= 3
    assert s["sm_mhz"] == statistics.median(float(l.split(",")[2]) for l in inside)
    assert s["sm_max_mhz"] == 1965 and s["reasons"] == []
    assert any(stamp(l) < c.t0 for l in c.lines)      # lead-in samples were taken and left out


def test_clock_sampler_reports_slowdown_and_short_regions(tmp_path):
    c = bench.Clocks(0, interval_ms=20, lead_s=0.6, smi=_fake_smi(tmp_path, slow_from=0))
    with c:
        pass                                 # shorter than one interval
    s = c.summary()
    assert s["samples"] == 1 and s["window"].startswith("nearest sample")
    assert s["reasons"] == ["hw_slowdown"]


def test_clock_sampler_targets_the_pci_address(tmp_path, monkeypatch):
    import types
    props = types.SimpleNamespace(pci_domain_id=0xABCD, pci_bus_id=0x3B, pci_device_id=0)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda i: props)
    assert bench.Clocks(0, smi=_fake_smi(tmp_path)).target() == "0000ABCD:3B:00.0"
    props.pci_bus_id = 0x3C                   # unknown to nvidia-smi: fall back to the index
    assert bench.Clocks(0, smi=_fake_smi(tmp_path)).target() == "0"


def test_clock_sampler_without_nvidia_smi():
    c = bench.Clocks(0, smi="/nonexistent/nvidia-smi")
    with c:
        pass
    s = c.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and s["window"] == "no samples"


def test_native_line_carries_the_contract():
    """The native arm's JSON line from measured numbers (those of a B200 run):
    every key of the contract, the roofline fraction from the algorithmic bytes
    and the kernel time, and the cpu_baseline when rank 0 timed the oracle."""
    import dataclasses
    from sparse_long_context_min_b200 import workloads
    cfg = dataclasses.replace(workloads.config(4), lengths=[1 << 20])
    stage = {"append": 9.6, "score": 28.8, "select": 16.4, "attend": 47.3}
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 12, "window": "timed region"}
    cpu = {"value": 378791.7, "unit": "us/step", "cores": 1, "kind": "oracle", "sample": "kv head 0"}
    line = bench.native_line(cfg, 1, 20, 5, 88.19, 86.0, 88.0, 28.78, stage, 2056, 278.2, {"x": 1},
                             (100.91, 20480, 16384), clk, cpu, (6528.7, "measured"), attend_us=21.5)
    json.loads(json.dumps(line))
    assert {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
            "cpu_baseline"} <= set(line)
    assert line["value"] == 88.19 and line["higher_is_better"] is False and line["scaling"] == "weak"
    assert line["gpu_launches"] == 4 * 20 and line["config"]["x"] == 1
    r = line["roofline"]                         # the dominant kernel: the fused attention, on the bytes it must read
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r)
    by = bench.algorithmic_bytes(cfg, 2056, 278.2, "topk")
    assert abs(r["achieved"] - by["attend"] / 21.5e-6 / 1e9) < 0.1
    assert abs(r["frac"] - r["achieved"] / 6528.7) < 1e-3
    assert abs(r["frac_of_8tbs"] - r["achieved"] / 8000.0) < 1e-3
    assert r["traffic"] == bench.ATTEND_DRAM_BYTES_1M and r["bytes_per_launch"] == by["attend"]
    rs = line["roofline_score"]                  # the scoring kernel with the token append
    assert abs(rs["achieved"] - by["score"] / 28.78e-6 / 1e9) < 0.1
    assert rs["traffic"] == round(bench.SCORE_DRAM_BYTES_PER_ROW * 16384 * 8)
    assert line["e2e"] == {"value": 100.91, "unit": "us/step", "h2d_bytes_per_step": 20480,
                           "d2h_bytes_per_step": 16384}
    assert line["config"]["step_us_best"] == 86.0 and line["config"]["workload"] == bench.workload_name(1 << 20)
    other = bench.native_line(cfg, 2, 20, 5, 88.19, 86.0, 88.0, 28.78, stage, 2056, 278.2,
                              {}, (100.91, 20480, 16384), clk, None, (6650.0, "fallback"), 21.5)
    assert "cpu_baseline" not in other and other["roofline"]["peak_kind"] == "fallback"
    short = dataclasses.replace(cfg, lengths=[1 << 18])   # the ncu traffic figure is of the 2^20 launch only
    assert bench.native_line(short, 1, 20, 5, 60.0, 58.0, 60.0, 10.0, stage, 520, 159.0, {},
                             (70.0, 20480, 16384), clk, None, (6528.7, "measured"), 15.0)["roofline"]["traffic"] is None


def test_oracle_leg_on_the_host_cores():
    """The cpu_baseline leg runs the oracle in a process without a GPU: one
    core, then one worker process per kv head (up to the host's cores), and
    the full-cache decode of one kv head; a small context keeps it short."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "bench.py", "--oracle-leg", "--context", "65536", "--leg-seconds", "0.2"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert d["kind"] == "oracle" and d["unit"] == "us/step" and d["value"] > 0
    assert d["cores"] == min(8, len(os.sched_getaffinity(0))) and d["host_cores"] == len(os.sched_getaffinity(0))
    assert d["single_core_us_per_step"] > 0 and d["full_cache_us_per_step_single_core"] > 0
    assert "65536 tokens" in d["sample"]
