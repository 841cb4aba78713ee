"""Benchmark of the dense-and-sparse quantized GEMV on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c2] [--batch 1]
                    [--impl dsq|reference]

A step is one dsq_gemv call: the whole hot path (decode of the packed codes,
fp32 dot products, the fused CSR outlier pass, one fp16 store of y) over one
batch of the workload.  Default workload: the 11008x4096 3-bit affine
group-16 layer with 1% structured outliers at batch 1.

Device timing: the K timed calls are captured into CUDA graphs and replayed
between CUDA events on the launching stream, after W warm-up calls, with a
barrier and a device synchronise on both sides.  Consecutive calls rotate
over enough independent packed copies of the layer that the bytes touched
between two uses of one copy exceed twice the L2 size, so weights come from
HBM.  Under torchrun every rank runs its own copy of the workload (weak
scaling, no data-path collective) and the slowest rank's time is reported.

Printed: one JSON line on rank 0.
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
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("dense+sparse 3-bit GEMV µs/call and GB/s as fraction of HBM peak (1×B200)")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e nominal (~8 TB/s)


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--config", default="c2")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--impl", default="dsq", choices=["dsq", "reference"])
    ap.add_argument("--op", default="gemv", choices=["gemv", "decompose"],
                    help="decompose: time the on-device decomposition of the config's weights instead")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=200)
    return ap.parse_args(argv)


# ------------------------------------------------------------------ ranks

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_group(world: int, backend: str):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max_sum(dist, t_ms: float, units: float, device=None):
    """(max of t_ms, sum of units) over ranks; identity without a group."""
    if dist is None:
        return t_ms, units
    import torch
    a = torch.tensor([t_ms], dtype=torch.float64, device=device)
    b = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(a, op=dist.ReduceOp.MAX)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(a.item()), float(b.item())


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ peaks, clocks

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Polls NVML (SM clock, max SM clock, throttle reasons) in a thread."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting"}

    def __init__(self, index: int, period_s: float = 0.001):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = get(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml" if self.nv else "unavailable"}


# ------------------------------------------------------------------ traffic record

def strip_comments(src: str) -> str:
    """C/C++ source without its // and /* */ comments (string and character
    literals kept), whitespace-normalised per line."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (" ".join(line.split()) for line in "".join(out).splitlines())
    return "\n".join(line for line in lines if line)


def kernel_source_digest(files=None) -> str:
    """Digest of library sources without their comments (all of them, or the
    named files of the csrc folder); a recorded ncu traffic figure only holds
    for the code it was measured on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dense_sparse_quantized_b200", "csrc")
    names = files if files else [n for n in os.listdir(csrc) if n.endswith((".cu", ".h"))]
    for name in sorted(names):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(config: str, batch: int):
    """ncu DRAM bytes per launch for (config, batch) from profiles/traffic.json,
    or None when absent or measured on other sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
        e = rec.get(f"{config}_b{batch}")
        if e and e.get("source_digest") == kernel_source_digest(e.get("sources")):
            return float(e["dram_bytes_per_launch"]), e.get("note", "")
    except Exception:
        pass
    return None, None


# ------------------------------------------------------------------ CPU oracle

def cpu_info():
    """(logical CPUs usable by this process, CPU model string)."""
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except Exception:
        pass
    return n, model


def oracle_rate(p, seconds: float, rows=None, threads: int = 1, x=None):
    """Time the oracle (decode + CSR + fp64 product) on host cores: repeated
    calls over `rows` (all rows by default) until `seconds` elapse.  With
    threads > 1 the rows are cut into `threads` contiguous slices that the
    unmodified single-threaded oracle computes concurrently (its C entry
    point releases the GIL).  Returns (GB/s on canonical bytes of the rows
    covered, calls, seconds)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    orc = oracle.load()
    rows = np.arange(p.rows, dtype=np.int32) if rows is None else np.asarray(rows, dtype=np.int32)
    frac = len(rows) / p.rows
    bytes_call = p.canonical_bytes(p.batch) * frac
    slices = [s for s in np.array_split(rows, max(1, threads)) if s.size]
    xv = p.x[:p.batch] if x is None else x
    with ThreadPoolExecutor(max_workers=len(slices)) as pool:
        t0 = time.perf_counter()
        n = 0
        while True:
            list(pool.map(lambda r: orc.gemv(p, x=xv, rows=r), slices))
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    return bytes_call * n / el / 1e9, n, el


def gpu_config(args, p, canon):
    """The workload keys both arms report."""
    import synth
    return {"workload": f"{args.config}: {synth.describe(args.config)}", "batch": args.batch,
            "rows": p.rows, "cols": p.cols, "bits": p.bits, "mode": p.mode, "nnz": p.nnz,
            "canonical_bytes_per_call": canon}


def run_reference(args):
    """The oracle, as it stands, on the host: one step = the oracle over a
    fixed row sample of the workload, computed by the unmodified
    single-threaded oracle on every host core (row slices in threads)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    import synth
    p = synth.make_config(args.config, batch=args.batch)
    orc = oracle.load()
    ncpu, model = cpu_info()
    rows = np.arange(0, p.rows, 16, dtype=np.int32)
    frac = len(rows) / p.rows
    canon = p.canonical_bytes(args.batch)
    bytes_step = canon * frac
    slices = [r for r in np.array_split(rows, ncpu) if r.size]
    from concurrent.futures import ThreadPoolExecutor
    xv = p.x[:args.batch]
    with ThreadPoolExecutor(max_workers=len(slices)) as pool:
        step = lambda: list(pool.map(lambda r: orc.gemv(p, x=xv, rows=r), slices))  # noqa: E731
        for _ in range(args.warmup):
            step()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            step()
        el = time.perf_counter() - t0
    ms = el / args.steps * 1e3
    gbs = bytes_step / (el / args.steps) / 1e9
    sample = (f"every 16th output row ({len(rows)} of {p.rows}) of {args.config} per step, "
              f"batch {p.batch}; bytes scaled to those rows; the single-threaded oracle on "
              f"{len(slices)} row slices in parallel threads")
    line = {"metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "us_per_call_full_layer": ms * 1e3 / frac, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": gpu_config(args, p, canon),
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": len(slices), "kind": "oracle",
                             "sample": sample, "nproc": ncpu, "cpu_model": model},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

def run_dsq(args):
    import torch
    import dense_sparse_quantized_b200 as dsq
    import synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_group(world, "nccl")

    p = synth.make_config(args.config, batch=args.batch)
    blob = dsq.pack_problem(p)
    canon = p.canonical_bytes(args.batch)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    first = dsq.Handle(blob, device=local)
    dev_bytes = first.device_bytes
    per_call = dev_bytes + args.batch * (p.cols + p.rows) * 2
    copies = max(2, math.ceil(2 * l2 / per_call) + 1)
    handles = [first] + [dsq.Handle(blob, device=local) for _ in range(copies - 1)]
    x_host = torch.from_numpy(p.x[:args.batch].view(np.int16)).view(torch.float16)
    xs = [x_host.to(device) for _ in range(copies)]
    ys = [torch.empty((args.batch, p.rows), dtype=torch.float16, device=device)
          for _ in range(copies)]
    launches_per_call = handles[0].launches_per_call(args.batch)

    stream = torch.cuda.Stream(device=device)

    def call(i):
        handles[i % copies].gemv(xs[i % copies], ys[i % copies], stream=stream)

    # warm-up (plain launches)
    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            call(i)
    stream.synchronize()

    # capture the K timed calls as graphs of G calls (G a multiple of copies,
    # about 120 calls, so the replays also give a per-call distribution)
    K = args.steps
    G = min(K, copies * max(1, 120 // copies))
    graphs = []
    with torch.cuda.stream(stream):
        for start in range(0, K, G):
            n = min(G, K - start)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    call(i)
            graphs.append(g)
    stream.synchronize()
    with torch.cuda.stream(stream):   # replays launch on the current stream
        for g in graphs:              # one untimed replay of every graph
            g.replay()
    stream.synchronize()

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    marks = [torch.cuda.Event(enable_timing=True) for _ in graphs]
    barrier(dist, device)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks, torch.cuda.stream(stream):
        ev0.record(stream)
        for g, mk in zip(graphs, marks):
            g.replay()
            mk.record(stream)
        ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize()
    barrier(dist, device)
    t_ms = ev0.elapsed_time(ev1)
    # per-call time of each replay (calls of one graph, back to back)
    sizes = [min(G, K - s0) for s0 in range(0, K, G)]
    per_replay, prev = [], ev0
    for mk, n in zip(marks, sizes):
        per_replay.append(prev.elapsed_time(mk) * 1e3 / n)
        prev = mk

    # latency of one isolated call on the device: a short device-side sleep
    # holds the stream while the host enqueues the events and the call, so
    # the call neither overlaps a neighbouring call nor waits for the host
    iso = []
    with torch.cuda.stream(stream):
        for i in range(60):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            stream.synchronize()
            torch.cuda._sleep(200000)   # ~0.1 ms of device time
            a.record(stream)
            call(i)
            b.record(stream)
            b.synchronize()
            if i >= 10:
                iso.append(a.elapsed_time(b) * 1e3)
    for h in handles:
        h.check()     # raises if a kernel gave up a bounded wait
    t_max, units = reduce_max_sum(dist, t_ms, canon * K, device)

    us_call = t_ms * 1e3 / K
    value = units / (t_max * 1e-3) / 1e9               # whole-job GB/s
    peak, peak_src = measured_peaks()
    achieved = canon / (us_call * 1e-6) / 1e9
    traffic, traffic_note = recorded_traffic(args.config, args.batch)

    # ---- end to end through the public API with host buffers
    e2e_steps = max(10, args.e2e_steps)
    x_pin = x_host.pin_memory()
    y_pin = torch.empty((args.batch, p.rows), dtype=torch.float16).pin_memory()
    xd = torch.empty_like(xs[0])
    yd = torch.empty_like(ys[0])
    with torch.cuda.stream(stream):
        for _ in range(3):
            handles[0].gemv_host(x_pin, y_pin, xd, yd, stream=stream)
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e2e_steps):
            handles[i % copies].gemv_host(x_pin, y_pin, xd, yd, stream=stream)
        e1.record(stream)
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_max, e2e_units = reduce_max_sum(dist, e2e_ms, canon * e2e_steps, device)
    e2e_value = e2e_units / (e2e_max * 1e-3) / 1e9

    # ---- CPU baseline: the oracle as it stands, rank 0, N = 1 only: on one
    # core, and on every core (row slices computed by the single-threaded
    # oracle in parallel threads)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ncpu, model = cpu_info()
        gbs1, n1, el1 = oracle_rate(p, 8.0)
        gbs, n, el = oracle_rate(p, 8.0, threads=ncpu)
        cpu = {"value": gbs, "unit": "GB/s", "cores": ncpu, "kind": "oracle",
               "sample": f"{n} full {args.config} oracle calls at batch {args.batch} "
                         f"({el:.1f} s) on {ncpu} row slices in parallel threads",
               "nproc": ncpu, "cpu_model": model,
               "single_core": {"value": gbs1, "unit": "GB/s", "cores": 1,
                               "sample": f"{n1} full calls ({el1:.1f} s, one thread)",
                               "us_per_call": el1 / n1 * 1e6},
               "us_per_call": el / n * 1e6}

    n_graphs = len(graphs)
    del graphs
    for h in handles:
        h.close()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": t_max / K,
            "us_per_call": us_call, "frac_of_hbm": achieved / peak,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16 in / f32 accumulate / f16 out", "data": "synthetic",
            "config": {**gpu_config(args, p, canon),
                       "device_bytes_per_call": per_call,
                       "l2": f"rotating {copies} packed copies "
                             f"({copies * per_call / 1e6:.0f} MB > 2x L2 {l2 / 1e6:.0f} MB)",
                       "timing": f"CUDA events around {n_graphs} CUDA graph replay(s) "
                                 f"of {K} calls"},
            "us_per_call_dist": {"median": float(np.median(per_replay)),
                                 "p10": float(np.percentile(per_replay, 10)),
                                 "p90": float(np.percentile(per_replay, 90)),
                                 "samples": len(per_replay),
                                 "what": f"per-call time of each graph replay ({G} calls back to back)"},
            "isolated_us_per_call": {"median": float(np.median(iso)),
                                     "p10": float(np.percentile(iso, 10)),
                                     "p90": float(np.percentile(iso, 90)),
                                     "samples": len(iso),
                                     "what": "CUDA events around one call after a device-side "
                                             "sleep and nothing after it (no overlap with "
                                             "neighbouring calls, no host launch gap)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_src == "measured" else "fallback 6650 GB/s",
                         "achieved_on_device_bytes": per_call / (us_call * 1e-6) / 1e9,
                         "traffic_note": traffic_note},
            "e2e": {"value": e2e_value, "unit": "GB/s",
                    "h2d_bytes_per_step": int(x_pin.numel() * 2),
                    "d2h_bytes_per_step": int(y_pin.numel() * 2),
                    "us_per_step": e2e_max * 1e3 / e2e_steps,
                    "path": "Handle.gemv_host: pinned x -> device, dsq_gemv, y -> pinned host"},
            "gpu_launches": K * launches_per_call,
            "clocks": clocks.summary(),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_decompose(args):
    """The step before the product on one GPU: dsq_decompose of the config's
    shape from fp32 weights (N(0, 0.02^2) plus Laplace spikes) resident in
    HBM, the outlier count of the config, K timed calls between CUDA events."""
    import torch
    import dense_sparse_quantized_b200 as dsq
    import synth
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    c = synth.CONFIGS[args.config]
    if c["mode"] not in ("lut", "affine"):
        raise SystemExit("decompose covers table and affine configs")
    M, N, bits, mode = c["rows"], c["cols"], c["bits"], c["mode"]
    nnz = synth.round_half_up(c["density"] * M * N)
    w = torch.from_numpy(synth.spiky_weights(M, N, c["density"], c["seed"])).cuda()
    out = dsq.decompose(w, bits, mode, nnz)          # allocates outputs and workspace once
    ws_bytes = ctypes_workspace_bytes(dsq, M, N, bits, mode, nnz)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=w.device)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            dsq.decompose(w, bits, mode, nnz, stream=stream, workspace=ws)
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks, torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            dsq.decompose(w, bits, mode, nnz, stream=stream, workspace=ws)
        e1.record(stream)
        e1.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / args.steps
    table_b = M * (1 << bits) * 2 if mode == "lut" else M * (N // 16) * 4
    alg = 4 * M * N + M * N + table_b + 6 * nnz + 4 * (M + 1)
    peak, peak_src = measured_peaks()
    line = {"metric": "on-device dense-and-sparse decomposition: us per matrix, GB/s on W read once + arrays written",
            "value": alg / (us * 1e-6) / 1e9, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us / 1e3, "us_per_call": us, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 in / f64 quantizer arithmetic",
            "data": "synthetic",
            "config": {"workload": f"{args.config} shape: {M}x{N} {mode} {bits}-bit, {nnz} outliers "
                                   "(top |w|) from N(0,0.02^2) + Laplace(0,0.2) spikes",
                       "rows": M, "cols": N, "bits": bits, "mode": mode, "nnz": nnz,
                       "algorithmic_bytes": alg, "launches_per_call": 9 if nnz else 3,
                       "l2": "W (fp32) is %d MB; it is read by several passes per call" % (4 * M * N // 10**6)},
            "roofline": {"bound": "hbm", "achieved": alg / (us * 1e-6) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": alg / (us * 1e-6) / 1e9 / peak, "traffic": None,
                         "peak_source": peak_src},
            "clocks": clocks.summary()}
    del out
    print(json.dumps(line), flush=True)
    return 0


def ctypes_workspace_bytes(dsq, M, N, bits, mode, nnz):
    import ctypes
    d = dsq.Desc(M, N, bits, dsq.MODE_LUT_ROW if mode == "lut" else dsq.MODE_AFFINE_G16, nnz)
    size = ctypes.c_size_t(0)
    dsq.library().dsq_decompose(ctypes.byref(d), None, None, None, None, None, None, None, None,
                                ctypes.byref(size), None)
    return size.value


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "decompose":
        return run_decompose(args)
    return run_dsq(args)


if __name__ == "__main__":
    sys.exit(main())
