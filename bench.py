"""Throughput of the low-bit linear layer on B200.

One step = one pass of the hot path over the 4B-class ternary sweep: for both
matrices (2560->9728, 9728->2560) and every M in {8192, 1024, 128, 16, 1},
per-token int8 quantisation of bf16 activations followed by the ternary
linear with bf16 output (tensor-core GEMM for M > 16, packed-weight GEMV for
M <= 16).  Weights are packed once, off the timed path, into a pool of
copies larger than L2 that the launches rotate through, so each launch reads
its weights from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python bench.py --workload t4nt_int4

Prints one JSON line (rank 0).  ``value`` is int TOPS (2*M*N*K summed over
the step's linears, divided by the device time of the whole step, summed over
ranks); per-kernel figures come from CUDA events around each launch.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from binary_weight_transformer_b200 import workloads as wls  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 vs 2.25 PFLOP/s)
L2_BYTES = 126 * 2**20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(summary: str, source: str):
    """DRAM bytes per launch from a committed ncu summary under profiles/,
    or None when the kernel's source has changed since the capture."""
    import hashlib
    import re
    try:
        text = open(os.path.join(ROOT, "profiles", summary)).read()
        src = open(os.path.join(ROOT, "binary_weight_transformer_b200", "csrc", source), "rb").read()
    except OSError:
        return None
    sha = re.search(r"sha256 prefix ([0-9a-f]{16})", text)
    val = re.search(r"traffic_bytes_per_launch: (\d+)", text)
    if not sha or not val or hashlib.sha256(src).hexdigest()[:16] != sha.group(1):
        return None
    return int(val.group(1))


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def shard_range(M: int, rank: int, world: int):
    """Token rows [start, stop) of rank `rank` when M rows are split across
    `world` ranks as evenly as possible (per-token quantisation makes every
    row independent, so the shards need no exchange)."""
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks of the default process group (the
    whole-job time is the slowest rank's); returns `value` without a group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"lowbit_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                     hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        loaded = [r["sm"] for r in rows if r["power"] > 250.0] or [r["sm"] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
class Point:
    def __init__(self, mi, m, M, fmt, sm_count=148):
        import binary_weight_transformer_b200 as bwt
        self.mi, self.m, self.M = mi, m, M
        # the kernel lowbit_linear dispatches to, as the library reports it
        self.kernel = bwt.linear_kernel(M, m.N, m.K, fmt, 0, sm_count)
        # up to 16 tokens the packed weights dominate the bytes: HBM-bound
        self.bound = "hbm" if M <= 16 else "tensor"
        self.ops = 2 * M * m.N * m.K


def select_points(wl, only_M=None, sm_count=148):
    points = []
    for mi, m in enumerate(wl.matrices):
        for M in sorted(wl.Ms, reverse=True):
            if only_M is None or M in only_M:
                points.append(Point(mi, m, M, wl.fmt, sm_count))
    return points


def build_state(wl, device, pool_bytes_target, torch, bwt, only_M=None, pool_copies=None):
    """Pack the weights (off the timed path) into a rotating pool and create
    the activation, code and output buffers."""
    points = select_points(wl, only_M, torch.cuda.get_device_properties(device).multi_processor_count)
    packs = []
    for mi, m in enumerate(wl.matrices):
        w = torch.from_numpy(wls.workload_weights(wl, mi)).to(device)
        packed, s_w = bwt.lowbit_pack(w, wl.fmt, 1e-5)
        packs.append((packed, s_w))
        del w
    per_set = sum(p[0].numel() for p in packs)
    copies = pool_copies or max(2, int(np.ceil(pool_bytes_target / per_set)))
    # every launch of a step reads its own copy, so a step never re-reads
    # weights from L2: at least one copy per point
    pool = [[(p.clone(), s) for (p, s) in packs] for _ in range(copies)]
    xs, qs, sxs, ys = {}, {}, {}, {}
    for pt in points:
        key = (pt.mi, pt.M)
        x = wls.workload_activations(wl, pt.mi, pt.M)
        if wl.x_dtype == wls.BF16:
            xs[key] = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
        else:
            xs[key] = torch.from_numpy(x).to(device)
        qs[key] = torch.empty((pt.M, (pt.m.K + 15) // 16 * 16), dtype=torch.int8, device=device)
        sxs[key] = torch.empty(pt.M, dtype=torch.float32, device=device)
        ydt = torch.bfloat16 if wl.y_dtype == wls.BF16 else torch.float32
        ys[key] = torch.empty((pt.M, pt.m.N), dtype=ydt, device=device)
    torch.cuda.synchronize()
    return points, pool, xs, qs, sxs, ys


def run_gpu_arm(args, wl):
    import torch
    import binary_weight_transformer_b200 as bwt

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    ydt = bwt.BF16 if wl.y_dtype == wls.BF16 else bwt.F32
    only_M = set(int(v) for v in args.points.split(",")) if args.points else None
    points, pool, xs, qs, sxs, ys = build_state(wl, device, 3 * L2_BYTES, torch, bwt, only_M, args.pool_copies)
    stream = torch.cuda.current_stream()
    n_sets = len(pool)

    def step(s):
        """One pass of the hot path; weights come from pool set s (each point
        of the step reads its own copy)."""
        launches = 0
        for i, pt in enumerate(points):
            key = (pt.mi, pt.M)
            packed, s_w = pool[(s * len(points) + i) % n_sets][pt.mi]
            bwt.lowbit_act_quant(xs[key], 0.0, q=qs[key], s_x=sxs[key])
            # the act quant just before does not write the weights
            bwt.lowbit_linear(qs[key], sxs[key], packed, s_w, wl.fmt, pt.m.N, ydt, K=pt.m.K, y=ys[key],
                              weights_stable=True)
            launches += 2  # act quant + one linear kernel
        return launches

    # eager warm-up (sets kernel attributes, loads modules), then one captured
    # graph per timed step
    for w in range(args.warmup):
        step(w)
    torch.cuda.synchronize()
    graphs = []
    launches_per_step = 0
    for s_ in range(args.steps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            launches_per_step = step(s_)
        graphs.append(g)
    torch.cuda.synchronize()
    for w in range(min(args.warmup, len(graphs))):
        graphs[w].replay()
    torch.cuda.synchronize()

    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    for g in graphs:
        g.replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    launches = launches_per_step * args.steps
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), device)
    del graphs

    # Per-kernel device times: for each point, graphs of R back-to-back
    # launches of the act quant and of the linear kernel alone (weights still
    # rotating over the pool), timed by events around a replay.
    def timed_graph(fn, reps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(reps):
                fn(r)
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / reps

    per_point, per_act = [], []
    for i, pt in enumerate(points):
        key = (pt.mi, pt.M)
        reps = 4 if pt.M >= 4096 else 20
        per_act.append(timed_graph(lambda r: bwt.lowbit_act_quant(xs[key], 0.0, q=qs[key], s_x=sxs[key]), reps))
        per_point.append(timed_graph(
            lambda r: bwt.lowbit_linear(qs[key], sxs[key], pool[(i + r) % n_sets][pt.mi][0],
                                        pool[(i + r) % n_sets][pt.mi][1], wl.fmt, pt.m.N, ydt, K=pt.m.K,
                                        y=ys[key], weights_stable=True), reps))

    # end to end through the public API with host buffers (pinned), one replica
    e2e = None if args.no_e2e else run_e2e(args, wl, points, pool, qs, sxs, ys, torch, bwt, stream, ydt)

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return None

    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    int8_peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * INT8_OVER_BF16
    step_ops = sum(pt.ops for pt in points)
    ms_per_step = elapsed_ms / args.steps
    value = step_ops * world / (ms_per_step * 1e-3) / 1e12

    pts_out = []
    gemv_bytes = gemv_ms = 0.0
    big_ops = big_ms = 0.0
    xbytes = 2 if wl.x_dtype == wls.BF16 else 4
    for pt, ms, ams in zip(points, per_point, per_act):
        fmt_bits = {wls.TERNARY2: 2, wls.BINARY1: 1, wls.INT4: 4}[wl.fmt]
        packed_bytes = pt.m.N * pt.m.K * fmt_bits // 8
        act_bytes = pt.M * pt.m.K * (xbytes + 1) + 4 * pt.M
        d = {"matrix": f"{pt.m.K}->{pt.m.N}", "M": pt.M, "kernel": pt.kernel, "us": round(ms * 1e3, 2),
             "act_quant_us": round(ams * 1e3, 2),
             "act_quant_gbs": round(act_bytes / (ams * 1e-3) / 1e9, 1)}
        if pt.bound == "hbm":
            gbs = packed_bytes / (ms * 1e-3) / 1e9
            d.update(packed_gbs=round(gbs, 1), frac_hbm=round(gbs / hbm, 3))
            gemv_bytes += packed_bytes
            gemv_ms += ms
        else:
            tops = pt.ops / (ms * 1e-3) / 1e12
            d.update(int_tops=round(tops, 1), frac_int8=round(tops / int8_peak, 3))
            big_ops += pt.ops
            big_ms += ms
        pts_out.append(d)

    # dominant kernel: the tensor-core GEMM at the largest M (about 60% of the
    # step); the launch reported is the first matrix's, the one profiled
    big = [i for i, pt in enumerate(points) if pt.bound == "tensor"]
    dom_i = min(big, key=lambda i: (-points[i].M, i)) if big else max(range(len(points)), key=lambda i: per_point[i])
    dom, dom_ms = points[dom_i], per_point[dom_i]
    if dom.bound == "tensor":
        achieved = dom.ops / (dom_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(int8_peak, 1),
                    "unit": "TOPS", "frac": round(achieved / int8_peak, 4),
                    "traffic": profiled_traffic("gemm_pair_kernel_ternary_4b_M8192.md", "gemm_sm100.cu")
                    if (wl.name == "ternary_4b" and dom.M == 8192 and dom.mi == 0) else None,
                    "kernel": f"lowbit {dom.kernel}, M={dom.M} {dom.m.K}->{dom.m.N}",
                    "peak_note": f"int8 = 2 x bf16 sustained ({peak_kind})"}
    else:
        fmt_bits = {wls.TERNARY2: 2, wls.BINARY1: 1, wls.INT4: 4}[wl.fmt]
        byts = dom.m.N * dom.m.K * fmt_bits // 8
        achieved = byts / (dom_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved / hbm, 4), "traffic": None,
                    "kernel": f"lowbit {dom.kernel}, M={dom.M}", "peak_note": peak_kind}

    cpu = run_cpu_baseline(wl, args.cpu_seconds) if (rank == 0 and world == 1 and not args.no_cpu) else None
    line = {
        "metric": "low-bit linear int TOPS (M>=128) and GEMV packed-weight GB/s vs HBM roofline",
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8 x ternary -> int32 (bf16 in/out)" if wl.fmt == wls.TERNARY2 else "int8 x low-bit -> int32",
        "data": "synthetic (seeded N(0,1) activations with outliers, N(0,0.02) weights)",
        "config": {"workload": workload_name(wl, [pt.M for pt in points]),
                   "timing": "each timed step is a CUDA graph replay; per-kernel times from graphs of back-to-back "
                             "launches of one kernel (rotating weights), events around the replay",
                   "parallelism": f"replicas x{world} (token batches, no collective)",
                   "l2": f"weights rotate over {len(pool)} packed copies ({len(pool) * sum(p[0].numel() for p in pool[0]) / 2**20:.0f} MiB > L2); "
                         "activations at M=8192 exceed L2"},
        "int_tops_m_ge_128": round(big_ops / (big_ms * 1e-3) / 1e12, 1) if big_ms else None,
        "gemv_packed_gbs": round(gemv_bytes / (gemv_ms * 1e-3) / 1e9, 1) if gemv_ms else None,
        "points": pts_out,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    return line


def run_e2e(args, wl, points, pool, qs, sxs, ys, torch, bwt, stream, ydt):
    """Same step through the public API from pinned host buffers: H2D copy of
    each point's activations, act quant, linear, D2H copy of its output.  The
    copies run on their own streams (PCIe is full duplex), so one point's
    uploads and downloads overlap the kernels of the others; events order each
    buffer's reuse across steps."""
    host_x, dev_x, host_y = {}, {}, {}
    for pt in points:
        key = (pt.mi, pt.M)
        x = wls.workload_activations(wl, pt.mi, pt.M)
        if wl.x_dtype == wls.BF16:
            hx = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
        else:
            hx = torch.from_numpy(x).pin_memory()
        host_x[key] = hx
        dev_x[key] = torch.empty_like(hx, device=stream.device)
        host_y[key] = torch.empty(ys[key].shape, dtype=ys[key].dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host_x.values())
    d2h = sum(v.numel() * v.element_size() for v in host_y.values())
    up, down = torch.cuda.Stream(device=stream.device), torch.cuda.Stream(device=stream.device)
    ev = {name: {(pt.mi, pt.M): torch.cuda.Event() for pt in points}
          for name in ("x_ready", "x_free", "y_ready", "y_free")}
    started = set()
    counter = [0]

    def step():
        for pt in points:
            key = (pt.mi, pt.M)
            packed, s_w = pool[counter[0] % len(pool)][pt.mi]
            counter[0] += 1
            first = key not in started
            started.add(key)
            with torch.cuda.stream(up):
                if not first:
                    up.wait_event(ev["x_free"][key])      # previous step's act quant has read dev_x
                dev_x[key].copy_(host_x[key], non_blocking=True)
                ev["x_ready"][key].record(up)
            stream.wait_event(ev["x_ready"][key])
            bwt.lowbit_act_quant(dev_x[key], 0.0, q=qs[key], s_x=sxs[key], stream=stream)
            ev["x_free"][key].record(stream)
            if not first:
                stream.wait_event(ev["y_free"][key])      # previous step's download has read y
            bwt.lowbit_linear(qs[key], sxs[key], packed, s_w, wl.fmt, pt.m.N, ydt, K=pt.m.K, y=ys[key],
                              stream=stream, weights_stable=True)
            ev["y_ready"][key].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev["y_ready"][key])
                host_y[key].copy_(ys[key], non_blocking=True)
                ev["y_free"][key].record(down)

    steps = max(1, min(args.steps, 5))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(up)
    stream.wait_event(a)
    down.wait_event(a)
    for _ in range(steps):
        step()
    up.wait_stream(stream)
    up.wait_stream(down)
    b.record(up)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    ops = sum(pt.ops for pt in points)
    return {"value": round(ops / (ms * 1e-3) / 1e12, 2), "unit": "TOPS", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3), "steps": steps,
            "overlap": "H2D, kernels and D2H on three streams"}


# ---------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------
def workload_name(wl, Ms):
    """The workload as both arms report it: matrices and token counts."""
    return (f"{wl.name}: " + ", ".join(f"{m.K}->{m.N}" for m in wl.matrices)
            + f" x M in {sorted(set(Ms), reverse=True)}")


def oracle_sample_step(wl, rows_per_point, nthreads, cache):
    """One bounded step of the oracle: act quant -> add/sub/skip dot ->
    rescale for every point of the sweep, on the first `rows_per_point`
    tokens of each point.  Returns the int ops performed (2*rows*N*K)."""
    import oracle
    ops = 0
    for mi, m in enumerate(wl.matrices):
        if ("codes", mi) not in cache:
            codes, s_w = oracle.quantize(wls.workload_weights(wl, mi), wl.fmt, 1e-5)
            cache[("codes", mi)] = (codes, s_w)
        codes, s_w = cache[("codes", mi)]
        for M in sorted(wl.Ms, reverse=True):
            rows = min(M, rows_per_point)
            if ("x", mi, M) not in cache:
                cache[("x", mi, M)] = wls.workload_activations(wl, mi, M)
            x = cache[("x", mi, M)][:rows]
            q, s_x = oracle.act_quant(x, 0.0, bf16_bits=(wl.x_dtype == wls.BF16))
            acc = oracle.int_dot(q, codes, wl.fmt, nthreads=nthreads)
            oracle.rescale(acc, s_w, s_x, "bf16" if wl.y_dtype == wls.BF16 else "f32")
            ops += 2 * rows * m.N * m.K
    return ops


def run_cpu_baseline(wl, seconds_target):
    import oracle
    oracle.build()
    nthreads = oracle.max_threads()
    cache = {}
    rows = 1
    oracle_sample_step(wl, rows, nthreads, cache)  # warm: quantise weights
    # grow the sample until one step takes about a second
    while True:
        t0 = time.perf_counter()
        ops = oracle_sample_step(wl, rows, nthreads, cache)
        dt = time.perf_counter() - t0
        if dt > 1.0 or rows >= 8192:
            break
        rows *= 2
    total_ops, total_t, steps = 0, 0.0, 0
    while total_t < seconds_target:
        t0 = time.perf_counter()
        total_ops += oracle_sample_step(wl, rows, nthreads, cache)
        total_t += time.perf_counter() - t0
        steps += 1
    return {"value": round(total_ops / total_t / 1e12, 6), "unit": "TOPS", "cores": nthreads, "kind": "oracle",
            "sample": f"{steps} oracle steps, each the first {rows} token rows of every (matrix, M) point "
                      f"of {wl.name} (act quant, add/sub/skip int dot, rescale), {total_t:.1f} s"}


def run_reference_arm(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    oracle.build()
    nthreads = oracle.max_threads()
    cache = {}
    rows = 16
    oracle_sample_step(wl, rows, nthreads, cache)
    for _ in range(args.warmup):
        oracle_sample_step(wl, rows, nthreads, cache)
    t0 = time.perf_counter()
    ops = 0
    for _ in range(args.steps):
        ops += oracle_sample_step(wl, rows, nthreads, cache)
    dt = time.perf_counter() - t0
    value = ops / dt / 1e12
    sample = (f"each step: the first {rows} token rows of every (matrix, M) point of {wl.name} "
              f"(act quant, add/sub/skip int dot, rescale) on {nthreads} host threads")
    return {
        "impl": "reference",
        "metric": "low-bit linear int TOPS (M>=128) and GEMV packed-weight GB/s vs HBM roofline",
        "value": round(value, 6), "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int64 (oracle)", "data": "synthetic",
        "config": {"workload": workload_name(wl, wl.Ms),
                   "timing": f"host wall clock; each step a bounded sample (the first {rows} token rows of "
                             "every point)",
                   "parallelism": f"oracle on {nthreads} host threads"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": nthreads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lowbit", choices=["lowbit", "reference"])
    ap.add_argument("--workload", default="ternary_4b", choices=sorted(wls.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline leg")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--points", default=None, help="comma-separated subset of the sweep's M values")
    ap.add_argument("--pool-copies", type=int, default=None,
                    help="number of packed weight copies to rotate over (default: enough to exceed 3x L2)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = wls.WORKLOADS[args.workload]
    if args.impl == "reference":
        line = run_reference_arm(args, wl)
    else:
        line = run_gpu_arm(args, wl)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
