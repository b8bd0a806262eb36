"""Throughput of the low-bit linear layer on B200.

One step = one pass of the hot path over a workload's points (every matrix
at every token count M): the BitLinear call lowbit_bitlinear -- the
activation prologue (the workload's RMSNorm, gain or Hadamard rotation, if
any), per-token int8 quantisation, then the low-bit linear layer with the
workload's output dtype.  Up to 4 tokens the call is one fused kernel, and
all matrices at the same token count run as one grouped launch
(lowbit_bitlinear_group; --no-group: one call each); above, a prologue
kernel and the linear kernel.  The
default workload is the 4B-class ternary sweep (2560->9728 and 9728->2560,
M in {8192, 1024, 128, 16, 1}, bf16 in and out).  Weights are packed once,
off the timed path, into a pool of copies larger than L2 that the launches
rotate through, so each launch reads its weights from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python bench.py --workload t4nt_int4

Prints one JSON line (rank 0).  ``value`` is int TOPS: 2*M*N*K summed over
the step's linears and over ranks, divided by the device time of one step
(the slowest rank's).  Per-kernel figures come from CUDA events around
repeated graph replays of each kernel alone.  With ``--gpus N`` and no
torchrun environment, the script relaunches itself under
``torch.distributed.run`` with N ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import socket
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from binary_weight_transformer_b200 import workloads as wls  # noqa: E402

METRIC = "low-bit linear int TOPS (M>=128) and GEMV packed-weight GB/s vs HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 vs 2.25 PFLOP/s)
# tcgen05.mma kind::i8 issue rate measured back to back on one SM (int8 MACs
# per SM clock); x 2 ops x SMs x SM clock gives the tensor pipe's own bound.
I8_MAC_PER_CLK_SM = 8192
L2_BYTES = 126 * 2**20
FMT_BITS = {wls.TERNARY2: 2, wls.BINARY1: 1, wls.INT4: 4}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(key: str):
    """DRAM bytes per launch of a profiled kernel launch, from the
    machine-readable ncu summary profiles/roofline_traffic.json, or None when
    the kernel's source has changed since the capture (its sha256 prefix is
    recorded beside the figure) or the entry is missing."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "roofline_traffic.json")) as f:
            entry = json.load(f)[key]
        src = open(os.path.join(ROOT, "binary_weight_transformer_b200", "csrc", entry["source"]), "rb").read()
    except (OSError, KeyError, ValueError):
        return None
    if hashlib.sha256(src).hexdigest()[:16] != entry.get("source_sha256_16"):
        return None
    return int(entry["traffic_bytes_per_launch"])


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------
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


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_under_torchrun(nproc: int, argv) -> int:
    """Run this script with `nproc` ranks on this node (one per GPU) and
    return the launcher's exit status.  Rendezvous on 127.0.0.1; `timeout`
    bounds a rank that never joins."""
    cmd = ["timeout", "-k", "60", "1800", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd, cwd=ROOT)


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
# points of a workload and their rooflines
# ---------------------------------------------------------------------------
class Point:
    """One (matrix, M) of a workload, with its algorithmic work (stated per
    launch: ops = 2*M*N*K; bytes = packed weights + int8 codes and s_x read,
    weight scales read, y written)."""

    def __init__(self, wl, mi, m, M, rows, sm_count=148, fused=True):
        import binary_weight_transformer_b200 as bwt
        self.mi, self.m, self.M, self.rows = mi, m, M, rows
        self.kernel = bwt.linear_kernel(rows, m.N, m.K, wl.fmt, 0, sm_count)
        self.fused = bwt.bitlinear_fuses(rows, m.K, wl.hadamard, 0) and fused
        # decode points whose layers can share a grouped launch
        self.groupable = bwt.decodes_from_x(rows, m.K, wl.hadamard, 0)
        if self.fused:
            self.kernel = "gemv_group_kernel (fused prologue)"
        self.ops = 2 * rows * m.N * m.K
        ysz = 2 if wl.y_dtype == wls.BF16 else 4
        self.packed_bytes = m.N * m.K * FMT_BITS[wl.fmt] // 8
        sw_bytes = 4 if wl.fmt == wls.TERNARY2 else 4 * m.N
        self.bytes = self.packed_bytes + rows * m.K + 4 * rows + sw_bytes + rows * m.N * ysz
        xsz = 2 if wl.x_dtype == wls.BF16 else 4
        self.act_bytes = rows * m.K * (xsz + 1) + 4 * rows

    def bound(self, ridge: float) -> str:
        return "tensor" if self.ops / self.bytes > ridge else "hbm"


def select_points(wl, only_M=None, sm_count=148, rank=0, world=1, shard=False, fused=True):
    points = []
    for mi, m in enumerate(wl.matrices):
        for M in sorted(wl.Ms, reverse=True):
            if only_M is None or M in only_M:
                rows = M
                if shard:
                    a, b = shard_range(M, rank, world)
                    rows = b - a
                if rows > 0:
                    points.append(Point(wl, mi, m, M, rows, sm_count, fused))
    return points


def pack_matrix(wl, mi, device, torch, bwt):
    """Packed weights and per-row or per-tensor scales of matrix mi, with the
    workload's quantiser: the format's default, BitNet v1 centred sign codes,
    or sign codes whose per-row scale is OneBit's output value vector."""
    w = torch.from_numpy(wls.workload_weights(wl, mi)).to(device)
    if wl.quantizer == "centred":
        packed, s_w = bwt.lowbit_pack_ex(w, wl.fmt, bwt.QUANT_BINARY_CENTRED)
    else:
        packed, s_w = bwt.lowbit_pack(w, wl.fmt, 1e-5)
    if wl.quantizer == "onebit":
        s_w = torch.from_numpy(wls.workload_output_vector(wl, mi)).to(device)
    return packed, s_w


def build_state(wl, points, device, pool_bytes_target, torch, bwt, pool_copies=None, row_offset=None):
    """Pack the weights (off the timed path) into a rotating pool and create
    the activation, code and output buffers of every point."""
    packs = []
    for mi, m in enumerate(wl.matrices):
        packs.append(pack_matrix(wl, mi, device, torch, bwt))
    per_set = sum(p[0].numel() for p in packs)
    copies = pool_copies or max(2, int(np.ceil(pool_bytes_target / per_set)))
    pool = [[(p.clone(), s) for (p, s) in packs] for _ in range(copies)]
    xs, qs, sxs, ys = {}, {}, {}, {}
    gains = {}
    for mi in range(len(wl.matrices)):
        g = wls.workload_gain(wl, mi)
        gains[mi] = None if g is None else torch.from_numpy(g).to(device)
    for pt in points:
        key = (pt.mi, pt.M)
        x = wls.workload_activations(wl, pt.mi, pt.M)
        a = row_offset(pt.M) if row_offset else 0
        x = x[a:a + pt.rows]
        if wl.x_dtype == wls.BF16:
            xs[key] = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device).view(torch.bfloat16)
        else:
            xs[key] = torch.from_numpy(np.ascontiguousarray(x)).to(device)
        qs[key] = torch.empty((pt.rows, (pt.m.K + 15) // 16 * 16), dtype=torch.int8, device=device)
        sxs[key] = torch.empty(pt.rows, dtype=torch.float32, device=device)
        ydt = torch.bfloat16 if wl.y_dtype == wls.BF16 else torch.float32
        ys[key] = torch.empty((pt.rows, pt.m.N), dtype=ydt, device=device)
    torch.cuda.synchronize()
    return pool, xs, qs, sxs, ys, gains


def time_graph(torch, stream, fn, launches, reps):
    """Capture `launches` back-to-back calls of fn(r) into one CUDA graph,
    replay it `reps` times with events on the launching stream around each
    replay, and return the per-launch times in ms (one per replay)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for r in range(launches):
            fn(r)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    del g
    return [a.elapsed_time(b) / launches for a, b in evs]


def summary(ts):
    return {"median": statistics.median(ts), "min": min(ts), "n": len(ts)}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
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
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    shard = args.shard == "m"
    points = select_points(wl, only_M, sms, rank, world, shard, not args.unfused)
    offset = (lambda M: shard_range(M, rank, world)[0]) if shard else None
    pool, xs, qs, sxs, ys, gains = build_state(wl, points, device, 3 * L2_BYTES, torch, bwt, args.pool_copies,
                                               offset)
    stream = torch.cuda.current_stream()
    n_sets = len(pool)
    norm = bwt.NORM_RMS if wl.norm else bwt.NORM_NONE

    def bitlinear(pt, packed, s_w, x=None, stream_=None):
        """The point's whole BitLinear call; the codes stay in the fused
        kernel's shared memory, else they go through q and s_x."""
        key = (pt.mi, pt.M)
        if not pt.fused and bwt.bitlinear_fuses(pt.rows, pt.m.K, wl.hadamard, 0):
            # --unfused: the prologue kernel and the linear kernel, as above 4 tokens
            bwt.lowbit_act_quant_ex(xs[key] if x is None else x, gains[pt.mi], norm, 1e-5, wl.hadamard, q=qs[key],
                                    s_x=sxs[key], stream=stream_)
            bwt.lowbit_linear(qs[key], sxs[key], packed, s_w, wl.fmt, pt.m.N, ydt, K=pt.m.K, y=ys[key],
                              stream=stream_, weights_stable=True, exclusive=True)
            return 2
        bwt.lowbit_bitlinear(xs[key] if x is None else x, packed, s_w, wl.fmt, pt.m.N, ydt, gains[pt.mi], norm,
                             1e-5, wl.hadamard, y=ys[key], q=None if pt.fused else qs[key],
                             s_x=None if pt.fused else sxs[key], stream=stream_, weights_stable=True,
                             exclusive=True)
        return 1 if pt.fused else 2

    # Token counts whose points are all fused decode calls run as grouped
    # launches (lowbit_bitlinear_group, up to GROUP_MAX layers per launch)
    # unless --no-group; `calls` lists the points of each API call of a step.
    group_ms = set()
    if not args.no_group and not args.unfused:
        for M in sorted({pt.M for pt in points}):
            at = [pt for pt in points if pt.M == M]
            if len(at) > 1 and all(pt.groupable for pt in at):
                group_ms.add(M)
    calls = []
    for M in sorted(group_ms):
        at = [(i, pt) for i, pt in enumerate(points) if pt.M == M]
        calls += [at[c:c + bwt.GROUP_MAX] for c in range(0, len(at), bwt.GROUP_MAX)]
    calls += [[(i, pt)] for i, pt in enumerate(points) if pt.M not in group_ms]

    def run_call(call, weights, x=None, stream_=None):
        """One API call of a step: a single point's bitlinear, or a grouped
        launch; weights(i, pt) gives the (packed, s_w) copy to read."""
        if call[0][1].M not in group_ms:
            i, pt = call[0]
            key = (pt.mi, pt.M)
            return bitlinear(pt, *weights(i, pt), x=None if x is None else x[key], stream_=stream_)
        keys = [(pt.mi, pt.M) for _, pt in call]
        ws = [weights(i, pt) for i, pt in call]
        two = any(pt.m.K > bwt.FUSED_MAX_K for _, pt in call)
        bwt.lowbit_bitlinear_group([(xs if x is None else x)[k] for k in keys], [w[0] for w in ws],
                                   [w[1] for w in ws], wl.fmt, [pt.m.N for _, pt in call], ydt,
                                   [gains[pt.mi] for _, pt in call], norm, 1e-5, ys=[ys[k] for k in keys],
                                   qs=[qs[k] for k in keys] if two else None,
                                   s_xs=[sxs[k] for k in keys] if two else None,
                                   stream=stream_, weights_stable=True, exclusive=True)
        n_long = sum(1 for _, pt in call if pt.m.K > bwt.FUSED_MAX_K)
        return (1 if n_long < len(call) else 0) + 2 * n_long

    def prologue(pt):
        key = (pt.mi, pt.M)
        bwt.lowbit_act_quant_ex(xs[key], gains[pt.mi], norm, 1e-5, wl.hadamard, q=qs[key], s_x=sxs[key])

    # The linear kernel timed alone reads codes that no prologue rewrites in
    # between, so each point rotates over copies of its codes whose total
    # exceeds twice L2 (at least two): every launch reads its codes from HBM,
    # as it does in the step.
    code_pool = {}
    for pt in points:
        key = (pt.mi, pt.M)
        copies = max(2, min(8, int(np.ceil(2 * L2_BYTES / max(1, qs[key].numel())))))
        code_pool[key] = [(qs[key], sxs[key])] + [(qs[key].clone(), sxs[key].clone()) for _ in range(copies - 1)]

    def linear(pt, packed, s_w, r=0):
        key = (pt.mi, pt.M)
        q_r, s_x_r = code_pool[key][r % len(code_pool[key])]
        # the prologue kernel just before does not write the weights
        bwt.lowbit_linear(q_r, s_x_r, packed, s_w, wl.fmt, pt.m.N, ydt, K=pt.m.K, y=ys[key],
                          weights_stable=True, exclusive=True)

    def step(s):
        """One pass of the hot path; each point of step s reads its own pool
        copy of the weights."""
        launches = 0
        for call in calls:
            launches += run_call(call, lambda i, pt: pool[(s * len(points) + i) % n_sets][pt.mi])
        return launches

    # eager warm-up (sets kernel attributes, loads modules), then a few
    # captured step graphs (each with its own rotation of the weight pool)
    # replayed cyclically for the K timed steps
    for w in range(args.warmup):
        step(w)
    torch.cuda.synchronize()
    n_graphs = max(1, min(args.steps, args.step_graphs))
    graphs = []
    launches_per_step = 0
    for s_ in range(n_graphs):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            launches_per_step = step(s_)
        graphs.append(g)
    torch.cuda.synchronize()
    for w in range(args.warmup):
        graphs[w % n_graphs].replay()
    torch.cuda.synchronize()

    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    for s_ in range(args.steps):
        graphs[s_ % n_graphs].replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    launches = launches_per_step * args.steps
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), device)
    del graphs

    # Per-kernel device times: for each point, a graph of back-to-back
    # launches of its act quant alone and one of its linear alone (weights
    # still rotating over the pool), each replayed `kernel_reps` times.
    per_point, per_act, per_call = [], [], []
    for i, pt in enumerate(points):
        launches_g = 4 if pt.rows >= 4096 else 20
        per_act.append(summary(time_graph(torch, stream, lambda r: prologue(pt), launches_g, args.kernel_reps)))
        launches_l = max(launches_g, len(code_pool[(pt.mi, pt.M)]))  # every code copy in each replay
        per_point.append(summary(time_graph(
            torch, stream, lambda r: linear(pt, *pool[(i + r) % n_sets][pt.mi], r=r), launches_l, args.kernel_reps)))
        per_call.append(summary(time_graph(
            torch, stream, lambda r: bitlinear(pt, *pool[(i + r) % n_sets][pt.mi]), launches_g, args.kernel_reps)))

    # Whole stack per token count: one graph of every matrix's act quant and
    # linear at that M (the per-layer chain a decode or prefill pass runs).
    stacks = {}
    for M in sorted({pt.M for pt in points}, reverse=True):
        pts = [(i, pt) for i, pt in enumerate(points) if pt.M == M]

        def stack(r, M=M, pts=pts):
            if M in group_ms:
                for call in calls:
                    if call[0][1].M == M:
                        run_call(call, lambda i, pt: pool[(r * len(points) + i) % n_sets][pt.mi])
                return
            for i, pt in pts:
                bitlinear(pt, *pool[(r * len(points) + i) % n_sets][pt.mi])
        stacks[M] = summary(time_graph(torch, stream, stack, 1, max(10, args.kernel_reps // 2)))

    # end to end through the public API with host buffers (pinned)
    e2e = None if args.no_e2e else run_e2e(args, wl, points, calls, pool, run_call, ys, torch, stream)

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return None

    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    int8_burst = float(peaks["bf16_tflops"]) * INT8_OVER_BF16
    int8_sustained = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * INT8_OVER_BF16
    sm_mhz = (clocks or {}).get("sm_mhz") or 1965.0
    issue_tops = I8_MAC_PER_CLK_SM * 2 * sms * sm_mhz * 1e6 / 1e12
    ridge = int8_burst * 1e12 / (hbm * 1e9)
    step_ops = sum(pt.ops for pt in points)
    ms_per_step = elapsed_ms / args.steps
    value = step_ops * world / (ms_per_step * 1e-3) / 1e12

    pts_out = []
    gemv_bytes = gemv_ms = 0.0
    big_ops = big_ms = 0.0
    for pt, tk, ta, tc in zip(points, per_point, per_act, per_call):
        # the linear kernel's own time (from codes), or the fused call's
        ms = tc["median"] if pt.fused else tk["median"]
        bound = pt.bound(ridge)
        d = {"matrix": f"{pt.m.K}->{pt.m.N}", "M": pt.M, "kernel": pt.kernel, "bound": bound,
             "us": round(ms * 1e3, 2), "us_min": round((tc if pt.fused else tk)["min"] * 1e3, 2), "reps": tk["n"],
             "call_us": round(tc["median"] * 1e3, 2), "fused": pt.fused,
             "linear_from_codes_us": round(tk["median"] * 1e3, 2),
             "prologue_us": round(ta["median"] * 1e3, 2),
             "prologue_frac_hbm": round(pt.act_bytes / (ta["median"] * 1e-3) / 1e9 / hbm, 3)}
        if pt.rows != pt.M:
            d["rows_this_rank"] = pt.rows
        if bound == "hbm":
            gbs = pt.bytes / (ms * 1e-3) / 1e9
            d.update(gbs=round(gbs, 1), frac_hbm=round(gbs / hbm, 3))
            if pt.M <= 16:
                pgbs = pt.packed_bytes / (ms * 1e-3) / 1e9
                d.update(packed_gbs=round(pgbs, 1), frac_hbm_packed=round(pgbs / hbm, 3))
                gemv_bytes += pt.packed_bytes
                gemv_ms += ms
        else:
            tops = pt.ops / (ms * 1e-3) / 1e12
            d.update(int_tops=round(tops, 1), frac_int8_burst=round(tops / int8_burst, 3),
                     frac_i8_issue=round(tops / issue_tops, 3))
        if pt.M >= 128:
            big_ops += pt.ops
            big_ms += ms
        pts_out.append(d)

    # dominant kernel: the linear point with the largest share of the step
    dom_i = max(range(len(points)), key=lambda i: (per_point[i]["median"], -i))
    dom, dom_ms = points[dom_i], per_point[dom_i]["median"]
    if dom.fused:
        dom_ms = per_call[dom_i]["median"]
    key = f"{dom.kernel} {wl.name} M={dom.M} {dom.m.K}->{dom.m.N}"
    if dom.bound(ridge) == "tensor":
        achieved = dom.ops / (dom_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(int8_burst, 1),
                    "unit": "TOPS", "frac": round(achieved / int8_burst, 4),
                    "traffic": profiled_traffic(key) if dom.rows == dom.M else None,
                    "kernel": f"lowbit {key}",
                    "peak_note": f"int8 = 2 x bf16 burst ({peak_kind}); the kernel is timed alone in "
                                 "graphs of back-to-back launches",
                    "frac_sustained": round(achieved / int8_sustained, 4),
                    "frac_i8_issue_rate": round(achieved / issue_tops, 4),
                    "i8_issue_rate_tops": round(issue_tops, 1)}
    else:
        achieved = dom.bytes / (dom_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved / hbm, 4),
                    "traffic": profiled_traffic(key) if dom.rows == dom.M else None,
                    "kernel": f"lowbit {key}", "peak_note": peak_kind}

    cpu = run_cpu_baseline(wl, args.cpu_seconds) if (world == 1 and not args.no_cpu) else None
    n_pool = sum(p[0].numel() for p in pool[0])
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "strong" if shard else "weak",
        "vs_baseline": None,
        "dtype": {wls.TERNARY2: "int8 x ternary -> int32", wls.BINARY1: "int8 x binary -> int32",
                  wls.INT4: "int8 x int4 -> int32"}[wl.fmt]
                 + f" ({'bf16' if wl.x_dtype == wls.BF16 else 'f32'} in, "
                   f"{'bf16' if wl.y_dtype == wls.BF16 else 'f32'} out)",
        "data": "synthetic (seeded N(0,1) activations with outliers, N(0,0.02) weights)",
        "config": {"workload": workload_name(wl, [pt.M for pt in points]),
                   "timing": f"K timed steps replay {n_graphs} captured step graphs cyclically, events on the "
                             f"launching stream around all K ({elapsed_ms:.0f} ms); per-kernel times are the "
                             f"median of {args.kernel_reps} replays of a graph of back-to-back launches of one "
                             "kernel (rotating weights, and rotating activation codes > 2x L2 for the linear "
                             "kernels)",
                   "flags": "weights-stable and exclusive (every kernel on one stream)",
                   "parallelism": (f"token rows sharded over {world} ranks, no collective" if shard
                                   else f"replicas x{world} (token batches, no collective)"),
                   "l2": f"weights rotate over {len(pool)} packed copies ({len(pool) * n_pool / 2**20:.0f} MiB "
                         "> L2); the largest activations exceed L2"},
        "int_tops_m_ge_128": round(big_ops / (big_ms * 1e-3) / 1e12, 1) if big_ms else None,
        "gemv_packed_gbs": round(gemv_bytes / (gemv_ms * 1e-3) / 1e9, 1) if gemv_ms else None,
        "stack_us": {str(M): round(v["median"] * 1e3, 2) for M, v in stacks.items()},
        "decode_groups": [{"M": M, "layers": sum(1 for pt in points if pt.M == M),
                           "launches": sum((1 if any(pt.m.K <= bwt.FUSED_MAX_K for _, pt in c) else 0)
                                           + 2 * sum(1 for _, pt in c if pt.m.K > bwt.FUSED_MAX_K)
                                           for c in calls if c[0][1].M == M),
                           "fused_layers": sum(1 for pt in points if pt.M == M and pt.m.K <= bwt.FUSED_MAX_K),
                           "us": round(stacks[M]["median"] * 1e3, 2),
                           "packed_gbs": round(sum(pt.packed_bytes for pt in points if pt.M == M)
                                               / (stacks[M]["median"] * 1e-3) / 1e9, 1),
                           "frac_hbm_packed": round(sum(pt.packed_bytes for pt in points if pt.M == M)
                                                    / (stacks[M]["median"] * 1e-3) / 1e9 / hbm, 3)}
                          for M in sorted(group_ms)],
        "points": pts_out,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    return line


def run_e2e(args, wl, points, calls, pool, run_call, ys, torch, stream):
    """Same step through the public API from pinned host buffers: H2D copy of
    each point's activations, the API calls of the step (one per point, or
    one per decode group), D2H copy of every output.  The copies run on their
    own streams (PCIe is full duplex), so one call's uploads and downloads
    overlap the kernels of the others; events order each buffer's reuse
    across steps."""
    host_x, dev_x, host_y = {}, {}, {}
    for pt in points:
        key = (pt.mi, pt.M)
        x = np.ascontiguousarray(wls.workload_activations(wl, pt.mi, pt.M)[:pt.rows])
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
        for call in calls:
            keys = [(pt.mi, pt.M) for _, pt in call]
            weights = {}
            for i, pt in call:
                weights[i] = pool[counter[0] % len(pool)][pt.mi]
                counter[0] += 1
            first = keys[0] not in started
            started.update(keys)
            with torch.cuda.stream(up):
                for key in keys:
                    if not first:
                        up.wait_event(ev["x_free"][key])      # previous step's call has read dev_x
                    dev_x[key].copy_(host_x[key], non_blocking=True)
                    ev["x_ready"][key].record(up)
            for key in keys:
                stream.wait_event(ev["x_ready"][key])
                if not first:
                    stream.wait_event(ev["y_free"][key])      # previous step's download has read y
            run_call(call, lambda i, pt: weights[i], x=dev_x, stream_=stream)
            for key in keys:
                ev["x_free"][key].record(stream)
                ev["y_ready"][key].record(stream)
            with torch.cuda.stream(down):
                for key in keys:
                    down.wait_event(ev["y_ready"][key])
                    host_y[key].copy_(ys[key], non_blocking=True)
                    ev["y_free"][key].record(down)

    steps = max(1, min(args.steps, args.e2e_steps))
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
    mats = []
    for m in wl.matrices:
        s = f"{m.K}->{m.N}"
        if s not in mats:
            mats.append(s)
    return f"{wl.name}: " + ", ".join(mats) + f" x M in {sorted(set(Ms), reverse=True)}"


def oracle_codes(wl, mi):
    """The oracle's weight codes and scales of matrix mi, with the workload's
    quantiser."""
    import oracle
    w = wls.workload_weights(wl, mi)
    if wl.quantizer == "centred":
        codes, beta, _ = oracle.binary_centred_codes(w)
        return codes, np.full(w.shape[0], beta[0], np.float32)
    codes, s_w = oracle.quantize(w, wl.fmt, 1e-5)
    if wl.quantizer == "onebit":
        s_w = wls.workload_output_vector(wl, mi)
    return codes, s_w


def oracle_sample_step(wl, rows_per_point, nthreads, cache):
    """One bounded step of the oracle: activation prologue -> add/sub/skip
    dot -> rescale for every point of the workload, on the first `rows_per_point`
    tokens of each point.  Returns the int ops performed (2*rows*N*K)."""
    import oracle
    ops = 0
    for mi, m in enumerate(wl.matrices):
        if ("codes", mi) not in cache:
            cache[("codes", mi)] = oracle_codes(wl, mi)
        codes, s_w = cache[("codes", mi)]
        g = wls.workload_gain(wl, mi)
        for M in sorted(wl.Ms, reverse=True):
            rows = min(M, rows_per_point)
            if ("x", mi, M) not in cache:
                cache[("x", mi, M)] = wls.workload_activations(wl, mi, M)
            x = cache[("x", mi, M)][:rows]
            q, s_x = oracle.act_prologue(x, g, wl.norm, 1e-5, wl.hadamard, bf16_bits=(wl.x_dtype == wls.BF16))
            acc = oracle.int_dot(q, codes, wl.fmt, nthreads=nthreads)
            oracle.rescale(acc, s_w, s_x, "bf16" if wl.y_dtype == wls.BF16 else "f32")
            ops += 2 * rows * m.N * m.K
    return ops


def _timed_oracle(wl, rows, nthreads, cache, seconds):
    total_ops, total_t, steps = 0, 0.0, 0
    while total_t < seconds or steps == 0:
        t0 = time.perf_counter()
        total_ops += oracle_sample_step(wl, rows, nthreads, cache)
        total_t += time.perf_counter() - t0
        steps += 1
    return total_ops / total_t / 1e12, steps, total_t


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
        oracle_sample_step(wl, rows, nthreads, cache)
        dt = time.perf_counter() - t0
        if dt > 1.0 or rows >= 8192:
            break
        rows *= 2
    value, steps, total_t = _timed_oracle(wl, rows, nthreads, cache, seconds_target)
    # one thread, on a smaller sample of the same points
    rows1 = max(1, rows // max(1, nthreads))
    value1, steps1, t1 = _timed_oracle(wl, rows1, 1, cache, max(2.0, seconds_target / 4))
    return {"value": round(value, 6), "unit": "TOPS", "cores": nthreads, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{steps} oracle steps, each the first {rows} token rows of every (matrix, M) point "
                      f"of {wl.name} (activation prologue and codes, add/sub/skip int dot, rescale), {total_t:.1f} s",
            "single_thread": {"value": round(value1, 6), "unit": "TOPS", "cores": 1,
                              "sample": f"{steps1} oracle steps of the first {rows1} token rows of every point, "
                                        f"{t1:.1f} s"}}


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
              f"(activation prologue and codes, add/sub/skip int dot, rescale) on {nthreads} host threads")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6), "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int64 (oracle)", "data": "synthetic",
        "config": {"workload": workload_name(wl, wl.Ms),
                   "timing": f"host wall clock; each step a bounded sample (the first {rows} token rows of "
                             "every point)",
                   "parallelism": f"oracle on {nthreads} host threads"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": nthreads, "kind": "oracle",
                         "cpu_model": cpu_model(), "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="lowbit", choices=["lowbit", "reference"])
    ap.add_argument("--workload", default="ternary_4b", choices=sorted(wls.WORKLOADS))
    ap.add_argument("--shard", default="replica", choices=["replica", "m"],
                    help="replica: every rank runs the whole step (weak scaling); m: the token rows of every "
                         "point are split across ranks (strong scaling)")
    ap.add_argument("--step-graphs", type=int, default=8, help="distinct captured step graphs replayed cyclically")
    ap.add_argument("--kernel-reps", type=int, default=50, help="replays per per-kernel timing graph")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline leg")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--points", default=None, help="comma-separated subset of the sweep's M values")
    ap.add_argument("--unfused", action="store_true",
                    help="run the prologue kernel and the linear kernel also where one fused call would run")
    ap.add_argument("--no-group", action="store_true",
                    help="one call per fused decode point instead of one grouped launch per token count")
    ap.add_argument("--pool-copies", type=int, default=None,
                    help="number of packed weight copies to rotate over (default: enough to exceed 3x L2)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1 or args.steps < 1 or args.kernel_reps < 1:
        ap.error("--gpus, --steps and --kernel-reps must be positive")
    return args


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    args = parse_args(argv)
    _, world, _ = dist_env()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_under_torchrun(args.gpus, argv)
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        return 2
    wl = wls.WORKLOADS[args.workload]
    if args.impl == "reference":
        line = run_reference_arm(args, wl)
    else:
        line = run_gpu_arm(args, wl)
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
