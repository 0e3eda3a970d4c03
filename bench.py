"""Benchmark of the approximate-softmax attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--part all|fwd|bwd] [--maps LABEL,...]

Workload (one step, the default): the forward of the B=1, H=32, S=16384,
D=128 causal problem with peaked keys (1% of keys shifted +3 along a per-head
unit direction), in bf16 and in e4m3, once per map.  Maps anchored at the
row's final statistics (two sweeps): exact softmax, Rowmax-PoT, and
K-interval K in {4, 16} x {min-max, fixed window} x {interpolation, hard
rounding}; maps anchored at the running maximum (one sweep, labels
"_online"): the online softmax (the exact-exp comparator), Rowmax-PoT and the
four fixed-window K-interval maps -- 32 forwards.  ``value`` is the step's
algorithmic TFLOP/s (4*B*H*S^2*D per forward, halved for causal; the
statistics sweep of the two-sweep maps is not counted), whole job, inputs
resident in HBM.  Every input set (bf16 402 MB, e4m3 201 MB) is larger than
the 126 MB L2; smaller workloads rotate over device copies.

The line also carries per-map TFLOP/s and fractions of the measured dense
peaks (the burst figures, with the sustained bf16 figure beside them), the
roofline of the dominant kernel (CUDA events on the launching stream), the
oracle timed on the host cores on a bounded sample, an end-to-end number
through pinned host buffers, sampled SM clocks, the host-side latency of one
call, board energy per forward read from the NVML energy counter, and
secondary figures: the non-causal 8K shape (each map with its own roofline),
the causal 8K and 2K shapes, and the K-interval backward on the training
shape.

--part fwd / bwd runs only the headline forwards / only the training-shape
backward (for profiler captures of exactly those launches); --maps restricts
the forwards to the named labels.

With --gpus N (launched under torchrun) every rank runs the same per-rank
problem on its own GPU (data-parallel over independent batches; there is no
exchange step), timing is the max over ranks and ``value`` sums all ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

HEADLINE = {"s16k_causal": ("s16k_bf16_causal", "s16k_fp8_causal")}
EXTRA_WORKLOADS = ("s8k_fp8", "s8k_bf16", "s8k_fp8_causal", "s2k_bf16_causal")
MODE_NAMES = {0: "exact", 1: "kinterval", 2: "rowmax_pot"}
CALIB_NAMES = {0: "minmax", 1: "fixed_window"}
ROUND_NAMES = {0: "interp", 1: "hard"}
CSRC = os.path.join(ROOT, "approximate_softmax_attention_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "fwd_traffic.json")
L2_BYTES = 126 * 2 ** 20
METRIC = ("attn fwd TFLOPS & % of B200 tensor peak per softmax mode, causal/non-causal "
          "2K-16K")


def mode_label(m):
    mode, K, cal, rnd = m[:4]
    anchor = m[4] if len(m) > 4 else 0
    lab = ("kinterval_K%d_%s_%s" % (K, CALIB_NAMES[cal], ROUND_NAMES[rnd]) if mode == 1
           else MODE_NAMES[mode])
    return lab + ("_online" if anchor else "")


def step_maps(w):
    """The maps of one step on workload w: the workload's maps anchored at the
    final row statistics (two sweeps), then the one-sweep forms anchored at
    the running maximum: the online softmax (this build's exact-exp
    comparator), Rowmax-PoT, and every fixed-window K-interval map of the
    workload."""
    maps = [tuple(m) + (0,) for m in w.modes]
    maps.append((0, 4, 0, 0, 1))
    maps.append((2, 4, 0, 0, 1))
    for (mode, K, cal, rnd) in w.modes:
        if mode == 1 and cal == 1:
            maps.append((mode, K, cal, rnd, 1))
    return maps


def dtype_name(w):
    return "e4m3" if w.dtype == "fp8" else "bf16"


def fwd_flops(w):
    f = 4.0 * w.B * w.H * w.S * w.S * w.D
    return f / 2 if w.causal else f


def input_bytes(w):
    return 3 * w.B * w.H * w.S * w.D * (1 if w.dtype == "fp8" else 2)


def load_peaks():
    """Dense peaks from the measured MEASURED_PEAKS.json (bf16 burst and
    sustained, HBM copy), else the pool's earlier measurement (fallback)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    hbm=float(d["hbm_gbs"]), source="measured (MEASURED_PEAKS.json)")
    return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0,
                source="fallback (no MEASURED_PEAKS.json on this box)")


def measure_gemm_peaks(dev, n=8192, reps=30):
    """Dense GEMM throughput measured here, with CUDA events, burst (a short
    loop): bf16 torch.matmul and e4m3 torch._scaled_mm (cuBLASLt), n^3."""
    import torch
    out = {}
    g = torch.Generator(device="cpu").manual_seed(0)
    a = torch.randn(n, n, generator=g).to(dev, torch.bfloat16)
    b = torch.randn(n, n, generator=g).to(dev, torch.bfloat16)
    flops = 2.0 * n ** 3

    def timeit(fn):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return flops * reps / (e0.elapsed_time(e1) * 1e-3) / 1e12

    out["bf16_tflops"] = round(timeit(lambda: a @ b), 1)
    try:
        a8 = a.to(torch.float8_e4m3fn)
        b8 = b.to(torch.float8_e4m3fn).t()          # column-major second operand
        one = torch.ones((), device=dev, dtype=torch.float32)
        out["e4m3_tflops"] = round(timeit(lambda: torch._scaled_mm(
            a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)), 1)
        out["e4m3_method"] = ("torch._scaled_mm e4m3 x e4m3 -> bf16, %d^3, per-tensor scales, "
                              "%d reps after 5 warm-up, CUDA events" % (n, reps))
    except Exception as e:  # pragma: no cover - depends on the box's cuBLASLt
        out["e4m3_tflops"] = None
        out["e4m3_method"] = "unavailable: %s" % (str(e).splitlines()[0][:120],)
    del a, b
    torch.cuda.empty_cache()
    return out


def dtype_peaks(peaks, gemm):
    """(burst, sustained, source) per dtype name."""
    bf = (peaks["bf16"], peaks["bf16_sustained"], "bf16 " + peaks["source"])
    if gemm.get("e4m3_tflops"):
        r = peaks["bf16_sustained"] / peaks["bf16"]
        e4 = (gemm["e4m3_tflops"], gemm["e4m3_tflops"] * r,
              "e4m3 measured in this run (%s); sustained = burst x the bf16 sustained/burst "
              "ratio" % gemm["e4m3_method"])
    else:
        e4 = (2 * peaks["bf16"], 2 * peaks["bf16_sustained"],
              "e4m3 = 2 x bf16 (nominal ratio; no e4m3 GEMM could be timed)")
    return {"bf16": bf, "e4m3": e4}


def gpu_uuid(dev):
    """The device's UUID as nvidia-smi / NVML print it ("GPU-..."), so that
    they address the same physical GPU as CUDA; None if torch cannot say."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, uuid=None):
        self.gpu = uuid or str(gpu_index)
        self.proc = None
        self.path = os.path.join("/tmp", "qsm_clocks_%d_%d.csv" % (os.getpid(), gpu_index))

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu,
                                          "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, pw, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                    pw.append(float(parts[3]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_median": statistics.median(pw) if pw else None}


KERNEL_HEADERS = ("wmap.cuh", "sm100.cuh", "internal.h")


def source_sha(name):
    """sha256 prefix of a kernel source file and the headers it includes (the
    key of the traffic records)."""
    h = hashlib.sha256()
    for n in (name,) + KERNEL_HEADERS:
        with open(os.path.join(CSRC, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def record_traffic(csv_path, workload):
    """Write the DRAM bytes of one forward step into the traffic records
    (profiles/fwd_traffic.json), from an ncu CSV of `bench.py --part fwd
    --workload W` that captured exactly one step's launches (-s warmup*n -c n)
    with dram__bytes_read.sum, dram__bytes_write.sum, gpu__time_duration.sum.
    Entries of other workloads are kept only while their kernel sources are
    unchanged."""
    import csv
    import io
    from approximate_softmax_attention_b200 import inputs
    names = HEADLINE.get(workload, (workload,))
    order = [(w.name, mode_label(m)) for w in (inputs.WORKLOADS[n] for n in names)
             for m in step_maps(w)]
    txt = open(csv_path).read()
    rows = list(csv.DictReader(io.StringIO(txt[txt.find('"ID"'):])))
    per = {}
    for r in rows:
        d = per.setdefault(int(r["ID"]), {"kernel": r["Kernel Name"]})
        d[r["Metric Name"]] = float(r["Metric Value"].replace(",", ""))
    launches = [per[i] for i in sorted(per)]
    if len(launches) != len(order):
        raise SystemExit("expected %d launches (one step), found %d" % (len(order), len(launches)))
    srcs = {n: source_sha(n) for n in ("fwd.cu", "fwd_online.cu")}
    old = {}
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            old = json.load(f)
    keep = {}
    if old.get("sources") == srcs:
        keep = {k: v for k, v in old.get("entries", {}).items()
                if not any(k.startswith(n + "/") for n in names)}
    for (wname, label), d in zip(order, launches):
        online = label.endswith("_online")
        if ("qsm_fwd_online_kernel" in d["kernel"]) != online:
            raise SystemExit("launch order does not match the step: %s vs %s" % (label, d["kernel"]))
        rd, wr = d["dram__bytes_read.sum"], d["dram__bytes_write.sum"]
        keep["%s/%s" % (wname, label)] = {
            "dram_bytes_per_launch": int(rd + wr), "dram_read": int(rd), "dram_write": int(wr),
            "ncu_duration_ns": int(d["gpu__time_duration.sum"])}
    out = {"sources": srcs,
           "source": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,"
                     "gpu__time_duration.sum --clock-control none -k regex:qsm_fwd -s <warm-up "
                     "launches> -c <one step> on python bench.py --part fwd --workload <W> "
                     "--steps 1 --warmup <w>; recorded by bench.py --record-traffic",
           "entries": dict(sorted(keep.items()))}
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print("recorded %d launches of %s into %s" % (len(order), workload, TRAFFIC_FILE))


def traffic_for(workload_name, label):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel that ran the map (fwd_online.cu for the
    one-sweep maps, fwd.cu otherwise); else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    src = "fwd_online.cu" if label.endswith("_online") else "fwd.cu"
    if d.get("sources", {}).get(src) != source_sha(src):
        return None
    e = d.get("entries", {}).get("%s/%s" % (workload_name, label))
    return None if e is None else e.get("dram_bytes_per_launch")


# ------------------------------------------------------------ oracle timing

def _cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(workloads, budget_s=12.0, rows_per_map=256):
    """Time the CPU oracle on a bounded sample: for every (workload, map), the
    same number of query rows spread over the sequence of one head; the
    algorithmic FLOPs of exactly those rows (4 D per valid key) are counted."""
    import numpy as np
    import oracle
    from approximate_softmax_attention_b200 import inputs
    cases = [(w, m) for w in workloads for m in step_maps(w)]
    per_case = budget_s / len(cases)
    done_flops, t_total, rows_done = 0.0, 0.0, 0
    draws = {}
    for w, m in cases:
        if w.name not in draws:
            draws[w.name] = inputs.draw(1, 1, w.S, w.D, seed=w.seed, peaked=w.peaked,
                                        dtype=w.dtype)
        d = draws[w.name]
        mode, K, cal, rnd, anchor = m
        n = rows_per_map
        t_case = 0.0
        while True:
            rows = np.unique(np.linspace(0, w.S - 1, n).astype(np.int64))
            kw = dict(q_descale=d["q_descale"], k_descale=d["k_descale"],
                      v_descale=d["v_descale"], rows=rows, row_block=128)
            t0 = time.perf_counter()
            if anchor and mode != 0:
                oracle.attn_fwd_online(d["q"], d["k"], d["v"], w.causal, mode, K=K,
                                       rounding=rnd, **kw)
            else:
                oracle.attn_fwd(d["q"], d["k"], d["v"], w.causal, mode, K=K, calib=cal,
                                rounding=rnd, **kw)
            dt = time.perf_counter() - t0
            keys = (rows + 1).sum() if w.causal else len(rows) * w.S
            done_flops += 4.0 * w.D * float(keys)
            t_case += dt
            rows_done += len(rows)
            if t_case >= 0.5 * per_case or n >= w.S:
                break
            n = min(w.S, 2 * n)
        t_total += t_case
    names = sorted({w.name for w, _ in cases})
    return {"value": done_flops / t_total / 1e12, "unit": "TFLOP/s", "cores": _cpu_cores(),
            "kind": "oracle",
            "sample": "%d query rows (evenly spaced over S, one head) for each of the %d "
                      "(workload, map) forwards of the step (%s); %.1f s of host time"
                      % (rows_done // len(cases), len(cases), ", ".join(names), t_total),
            "seconds": t_total, "flops": done_flops}


# ------------------------------------------------------- multi-rank logic

def max_over_ranks(x, world, device="cpu"):
    """The slowest rank's value (every rank calls this, in the same order)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_rank_step, ms_per_step_max, world):
    """Whole-job TFLOP/s: every rank runs its own problem of the same size
    (independent batches), the job takes as long as the slowest rank."""
    return world * flops_per_rank_step / (ms_per_step_max * 1e-3) / 1e12


# ----------------------------------------------------------------- GPU arm

class Problem:
    """One workload resident on the device, with the calls of its maps."""

    def __init__(self, w, dev, qsm, inputs, maps=None):
        import torch
        self.w = w
        d = inputs.draw_workload(w)
        self.d = d
        # rotate over copies only when one input set would fit in L2
        ncopy = 1 if input_bytes(w) > L2_BYTES else 3
        self.q = [d["q"].to(dev) for _ in range(ncopy)]
        self.k = [d["k"].to(dev) for _ in range(ncopy)]
        self.v = [d["v"].to(dev) for _ in range(ncopy)]
        self.ncopy = ncopy
        B, H, S, D = w.shape
        self.O = torch.empty(B, H, S, D, dtype=torch.bfloat16, device=dev)
        self.LSE = torch.empty(B, H, S, dtype=torch.float32, device=dev)
        self.opts = [qsm.make_opts(dtype=qsm.DTYPE_FP8_E4M3 if w.dtype == "fp8" else 0,
                                   q_descale=d["q_descale"], k_descale=d["k_descale"],
                                   v_descale=d["v_descale"], anchor=anchor)
                     for anchor in (0, 1)]
        self.modes = [m for m in step_maps(w) if maps is None or mode_label(m) in maps]
        self.qsm = qsm
        self.i = 0

    def call(self, m, stream, O=None, q=None, k=None, v=None):
        mode, K, cal, rnd, anchor = m
        c = self.i % self.ncopy
        st = self.qsm.qsm_attn_fwd(q if q is not None else self.q[c],
                                   k if k is not None else self.k[c],
                                   v if v is not None else self.v[c],
                                   self.O if O is None else O, self.LSE, self.w.causal, mode, K,
                                   cal, rnd, 0, self.opts[anchor], stream)
        if st != 0:
            raise RuntimeError("qsm_attn_fwd: " + self.qsm.qsm_status_string(st))
        self.i += 1

    def label(self, m):
        return "%s/%s" % (dtype_name(self.w), mode_label(m))


def time_calls(calls, stream, steps, warmup):
    """Per-call CUDA-event times (ms) of `steps` passes over `calls`, after
    `warmup` passes; returns (per-call lists, total ms of the timed passes)."""
    import torch
    for _ in range(warmup):
        for fn in calls:
            fn()
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in calls] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(steps):
        for j, fn in enumerate(calls):
            ev[s][j][0].record(stream)
            fn()
            ev[s][j][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    per = [[ev[s][j][0].elapsed_time(ev[s][j][1]) for s in range(steps)]
           for j in range(len(calls))]
    return per, t0.elapsed_time(t1)


def map_entry(w, ms, pk):
    tf = fwd_flops(w) / (ms * 1e-3) / 1e12
    burst, sust, _ = pk[dtype_name(w)]
    return {"ms": round(ms, 4), "tflops": round(tf, 1), "frac_of_dtype_peak": round(tf / burst, 4),
            "frac_of_dtype_peak_sustained": round(tf / sust, 4),
            "frac_of_bf16_peak": round(tf / pk["bf16"][0], 4)}


def roofline_of(w, label, entry, pk):
    burst, sust, src = pk[dtype_name(w)]
    kern = "qsm_fwd_online_kernel" if label.endswith("_online") else "qsm_fwd_kernel"
    return {"bound": "tensor", "kernel": "%s (%s, %s)" % (kern, w.name, label),
            "achieved": entry["tflops"], "peak": round(burst, 1), "unit": "TFLOP/s",
            "frac": round(entry["tflops"] / burst, 4),
            "peak_sustained": round(sust, 1),
            "frac_of_sustained": round(entry["tflops"] / sust, 4),
            "peak_source": "burst: %s" % src,
            "algorithmic_flops_per_launch": fwd_flops(w),
            "ms_per_launch": entry["ms"],
            "traffic": traffic_for(w.name, label)}


def energy_per_forward(prob, m, stream, dev_index, uuid=None, min_s=1.0):
    """Board energy per forward (J) from the NVML total-energy counter, read
    around a loop of forwards (read-only; on a shared machine other users'
    work on other GPUs does not enter this GPU's counter)."""
    import torch
    try:
        import pynvml
        pynvml.nvmlInit()
        h = (pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid
             else pynvml.nvmlDeviceGetHandleByIndex(dev_index))
    except Exception:
        return None
    for _ in range(3):
        prob.call(m, stream)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0 = pynvml.nvmlDeviceGetTotalEnergyConsumption(h)
    n = 0
    while time.perf_counter() - t0 < min_s or n < 5:
        for _ in range(5):
            prob.call(m, stream)
        n += 5
        torch.cuda.synchronize()
    e1 = pynvml.nvmlDeviceGetTotalEnergyConsumption(h)
    dt = time.perf_counter() - t0
    return {"joules_per_forward": round((e1 - e0) * 1e-3 / n, 4), "forwards": n,
            "avg_power_w": round((e1 - e0) * 1e-3 / dt, 1)}


def run_ours(args):
    import torch
    import torch.distributed as dist
    from approximate_softmax_attention_b200 import inputs, qsm

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    gemm = measure_gemm_peaks(dev) if rank == 0 or world > 1 else {}
    pk = dtype_peaks(peaks, gemm)
    maps = set(args.maps.split(",")) if args.maps else None

    names = HEADLINE.get(args.workload, (args.workload,))
    wls = [inputs.WORKLOADS[n] for n in names]
    probs = [] if args.part == "bwd" else [Problem(w, dev, qsm, inputs, maps) for w in wls]
    calls, labels, owners = [], [], []
    for p in probs:
        for m in p.modes:
            calls.append(lambda p=p, m=m: p.call(m, stream))
            labels.append(p.label(m))
            owners.append((p, m))
    step_flops = sum(fwd_flops(p.w) for p, _ in owners)

    line = None
    if calls:
        if world > 1:
            dist.barrier()
        for fn in calls * args.warmup:
            fn()
        torch.cuda.synchronize()
        clocks = ClockSampler(local, gpu_uuid(dev))
        clocks.start()
        time.sleep(0.3)
        per, ms_total = time_calls(calls, stream, args.steps, 0)
        ck = clocks.stop()
        ms_total = max_over_ranks(ms_total, world, dev)
        ms_step = ms_total / args.steps
        value = weak_scaling_value(step_flops, ms_step, world)
        per_mode = {}
        for j, (p, m) in enumerate(owners):
            per_mode[labels[j]] = map_entry(p.w, sum(per[j]) / len(per[j]), pk)
        # host-side call latency (the pages' other figure): wall time of one
        # qsm_attn_fwd call through the binding (validation, three tensor-map
        # encodings, one launch; it does not wait for the kernel)
        for j, (p, m) in enumerate(owners):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            for _ in range(10):
                p.call(m, stream)
            per_mode[labels[j]]["host_call_us"] = round((time.perf_counter() - t0) / 10 * 1e6, 1)
            torch.cuda.synchronize()
        dom = max(range(len(owners)), key=lambda j: per_mode[labels[j]]["ms"])
        dp, dm = owners[dom]
        roof = roofline_of(dp.w, mode_label(dm), per_mode[labels[dom]], pk)
        roof["time_share_of_step"] = round(per_mode[labels[dom]]["ms"] / ms_step, 4)

        e2e = None if args.no_e2e else run_e2e(probs, owners, stream, dev, args, world)
        energy = None
        if not args.no_energy and rank == 0:
            # exact and Rowmax-PoT, two-sweep and one-sweep, each dtype: the
            # pages' comparison (board energy per forward at causal 16K)
            energy = {}
            for j, (p, m) in enumerate(owners):
                if m[0] in (0, 2):
                    energy[labels[j]] = energy_per_forward(p, m, stream, local, gpu_uuid(dev))
        line = {
            "metric": METRIC,
            "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "+".join(sorted({dtype_name(w) for w in wls}, key=["bf16", "e4m3"].index)),
            "data": "synthetic (seeded randn, peaked keys)",
            "config": {"workload": args.workload,
                       "shapes": {w.name: {"B": w.B, "H": w.H, "S": w.S, "D": w.D,
                                           "causal": w.causal, "dtype": dtype_name(w)}
                                  for w in wls},
                       "maps": labels, "step": "one forward per (dtype, map)",
                       "parallelism": "dp%d" % world,
                       "l2": "; ".join("%s inputs %.0f MB%s" % (
                           w.name, input_bytes(w) / 1e6,
                           " > 126 MB L2" if input_bytes(w) > L2_BYTES else
                           ", rotated over 3 device copies") for w in wls)},
            "per_mode": per_mode,
            "roofline": roof,
            "peaks": {"bf16_burst": pk["bf16"][0], "bf16_sustained": pk["bf16"][1],
                      "bf16_source": peaks["source"], "e4m3_burst": round(pk["e4m3"][0], 1),
                      "e4m3_source": pk["e4m3"][2], "gemm_measured_here": gemm},
            "cpu_baseline": None,
            "e2e": e2e,
            "gpu_launches": args.steps * len(calls),
            "clocks": ck,
            "energy_per_forward": energy,
        }

    extras = {}
    if args.part == "all" and not args.no_extra and rank == 0:
        extras.update(run_extra_forwards(dev, qsm, inputs, stream, pk))
    if args.part in ("all", "bwd") and not args.no_extra and rank == 0:
        extras["train_s1k_bwd"] = run_backward(dev, qsm, inputs, stream, pk,
                                               reps=args.bwd_reps)
        for wn in ("train_s1k_d128", "train_s1k_d128_fp8"):
            extras[wn + "_bwd"] = run_backward(dev, qsm, inputs, stream, pk,
                                               reps=args.bwd_reps, workload=wn)

    cpu = None
    if line is not None and rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(wls, budget_s=args.cpu_budget)
        cpu.pop("seconds", None)
        cpu.pop("flops", None)

    if rank == 0:
        if line is None:
            line = {"metric": METRIC, "part": args.part, "extra": extras}
        else:
            line["cpu_baseline"] = cpu
            line["extra"] = extras
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(probs, owners, stream, dev, args, world):
    """The same step end to end through the public binding: every step copies
    its inputs from pinned host memory and reads every forward's O back; the
    read-back of one map's O runs on a copy stream while the next map
    computes."""
    import torch
    from approximate_softmax_attention_b200 import qsm  # noqa: F401
    copy = torch.cuda.Stream(dev)
    host_in = {id(p): [p.d[n].pin_memory() for n in ("q", "k", "v")] for p in probs}
    dev_in = {id(p): [torch.empty_like(p.q[0]) for _ in range(3)] for p in probs}
    outs = [torch.empty_like(p.O) for p, _ in owners]
    host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    done = [torch.cuda.Event() for _ in owners]
    h2d = sum(t.numel() * t.element_size() for v in host_in.values() for t in v)
    d2h = sum(o.numel() * o.element_size() for o in outs)

    def step():
        for p in probs:
            for hsrc, ddst in zip(host_in[id(p)], dev_in[id(p)]):
                ddst.copy_(hsrc, non_blocking=True)
        for j, (p, m) in enumerate(owners):
            q, k, v = dev_in[id(p)]
            p.call(m, stream, O=outs[j], q=q, k=k, v=v)
            done[j].record(stream)
            copy.wait_event(done[j])
            with torch.cuda.stream(copy):
                host_out[j].copy_(outs[j], non_blocking=True)
        stream.wait_stream(copy)

    for _ in range(max(1, min(args.warmup, 2))):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(1, min(args.steps, 5))
    a.record(stream)
    for _ in range(n):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / n, world, dev)
    flops = sum(fwd_flops(p.w) for p, _ in owners)
    return {"value": round(weak_scaling_value(flops, ms, world), 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "steps": n, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "path": "qsm_attn_fwd through the ctypes binding; pinned host inputs copied in, "
                    "every O copied out on a second stream overlapping the next forward"}


def run_extra_forwards(dev, qsm, inputs, stream, pk):
    import torch
    extras = {}
    for name in EXTRA_WORKLOADS:
        w = inputs.WORKLOADS[name]
        p = Problem(w, dev, qsm, inputs)
        calls = [lambda m=m: p.call(m, stream) for m in p.modes]
        per, _ = time_calls(calls, stream, 10, 3)
        res = {}
        for j, m in enumerate(p.modes):
            e = map_entry(w, sum(per[j]) / len(per[j]), pk)
            e["roofline"] = roofline_of(w, mode_label(m), e, pk)
            res[mode_label(m)] = e
        extras[name] = {"shape": list(w.shape), "dtype": dtype_name(w), "causal": w.causal,
                        "per_mode": res, "reps": 10,
                        "l2": "inputs %.0f MB%s" % (input_bytes(w) / 1e6,
                                                    "" if input_bytes(w) > L2_BYTES else
                                                    ", rotated over 3 device copies")}
        del p
        torch.cuda.empty_cache()
    return extras


def run_backward(dev, qsm, inputs, stream, pk, reps=10, workload="train_s1k"):
    """Training shape: forward with statistics, then the backward (2.5 x the
    forward's algorithmic FLOPs), per (map, surrogate).  An e4m3 workload runs
    the backward of its e4m3 forward (bf16 passes, FLOPs counted the same)."""
    import torch
    tw = inputs.WORKLOADS[workload]
    td = inputs.draw_workload(tw)
    tq, tk, tv, tdo = (td[n].to(dev) for n in ("q", "k", "v", "dO"))
    desc = dict(q_descale=td["q_descale"], k_descale=td["k_descale"],
                v_descale=td["v_descale"])
    ws = torch.empty(qsm.qsm_attn_bwd_workspace_size(*tw.shape), dtype=torch.uint8, device=dev)
    res = {}
    for (mode, K, cal, rnd) in tw.modes:
        for surr in (qsm.SURR_PRE, qsm.SURR_POST):
            O_, L_, st_ = qsm.attention_forward(tq, tk, tv, True, mode, K, cal, rnd, stats=True,
                                                **desc)
            fn = (lambda: qsm.attention_backward(tq, tk, tv, O_, tdo, L_, st_, True, mode, K,
                                                 cal, rnd, surr, workspace=ws, **desc))
            per, _ = time_calls([fn], stream, reps, 3)
            ms = sum(per[0]) / len(per[0])
            tf = 2.5 * fwd_flops(tw) / (ms * 1e-3) / 1e12
            lab = "%s_%s" % (mode_label((mode, K, cal, rnd)), {1: "pre", 2: "post"}[surr])
            res[lab] = {"bwd_ms": round(ms, 4), "bwd_tflops": round(tf, 1),
                        "frac_of_bf16_peak": round(tf / pk["bf16"][0], 4)}
    return {"shape": list(tw.shape), "dtype": "bf16" if tw.dtype == "bf16" else
            "e4m3 inputs, bf16 passes", "causal": True,
            "flops": "2.5 x 4*B*H*S^2*D/2", "per_mode": res}


# ---------------------------------------------------------- reference arm

def run_reference(args):
    """The oracle (fp64, host cores) on the same step: each step is a bounded
    sample of query rows of every (workload, map) forward; ``value`` is the
    algorithmic TFLOP/s of the rows processed and ``ms_per_step`` the host
    time one step took."""
    from approximate_softmax_attention_b200 import inputs
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    names = HEADLINE.get(args.workload, (args.workload,))
    wls = [inputs.WORKLOADS[n] for n in names]
    budget = max(2.0, min(20.0, args.ref_budget / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(wls, budget_s=budget / 4, rows_per_map=32)
    flops, secs, last = 0.0, 0.0, None
    for _ in range(args.steps):
        r = oracle_sample(wls, budget_s=budget, rows_per_map=64)
        flops += r["flops"]
        secs += r["seconds"]
        last = r
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded randn, peaked keys)",
        "config": {"workload": args.workload,
                   "shapes": {w.name: {"B": w.B, "H": w.H, "S": w.S, "D": w.D,
                                       "causal": w.causal, "dtype": dtype_name(w)}
                              for w in wls},
                   "maps": ["%s/%s" % (dtype_name(w), mode_label(m)) for w in wls
                            for m in step_maps(w)],
                   "step": "a bounded sample of query rows of every (dtype, map) forward"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": last["cores"],
                         "kind": "oracle", "sample": last["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="s16k_causal")
    ap.add_argument("--part", choices=["all", "fwd", "bwd"], default="all")
    ap.add_argument("--maps", default=None, help="comma-separated map labels to run")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-energy", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-budget", type=float, default=100.0)
    ap.add_argument("--bwd-reps", type=int, default=10)
    ap.add_argument("--record-traffic", metavar="CSV", default=None,
                    help="write an ncu DRAM capture of one --part fwd step of --workload into "
                         "the traffic records and exit (no GPU needed)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.part != "all":
        args.no_e2e = args.no_energy = args.no_cpu_baseline = True
    if args.record_traffic:
        record_traffic(args.record_traffic, args.workload)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
