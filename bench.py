#!/usr/bin/env python
"""Benchmark: MoE layer forward (route + pack + compute + combine) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--also A,B,..]
                    [--impl ours|reference]

Headline workload (default): the largest single-GPU configuration, the 64 routed + 1 shared
expert layer (T=4096, d=4096, SwiGLU d_ff=32768, top-2, dropless, bf16; 52 GB of weights).
A step is one forward of the workload's layers (one layer here; the Granite-shaped stack has
24 chained by the residual).  The metric is routed tokens per second per MoE layer forward:
T * layers / step time, summed over ranks.  `value` and `ms_per_step` come from K replays of
the plain CUDA graph of the step, timed with CUDA events on the launching stream.  The
per-kernel times behind `roofline` and `kernels` come from a separate pass of replays whose
graphs carry an event between kernels (those events break the overlap of programmatic
dependent launches, so that pass is kept out of the timed region).  `workloads` repeats the
measurement on the other configurations: the Granite-shaped stack, the Mixtral-shaped
prefill and decode layers, the 64+1 decode layer, the Switch-shaped and the reroute layers.
With N > 1 each rank runs an independent replica (weak scaling, no collective on the data
path).  Prints one JSON line (rank 0).

--impl reference times the fp64 CPU oracle on the host cores (a bounded sample per step).
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed tokens/s per MoE layer fwd (1×B200) + % of bf16 TC / HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Specification figures the metric is also quoted against: dense bf16 tensor throughput and
# HBM3e bandwidth of one B200.
SPEC_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}
KERNELS = ["route", "pack", "gemm_gate_up", "gemm_down", "combine"]
KERNEL_SOURCES = {"route": ["route.cu", "route_sm100.cu", "dispatch_prep.cuh", "common.cuh"],
                  "pack": ["dispatch.cu", "dispatch_prep.cuh", "reroute.cu", "common.cuh"],
                  "gemm_gate_up": ["gemm_sm100.cu", "gemm_cols_sm100.cu", "gemm_pair_sm100.cu",
                                   "gemm_rowpair_sm100.cu", "gemm_common.cuh", "common.cuh"],
                  "gemm_down": ["gemm_sm100.cu", "gemm_cols_sm100.cu", "gemm_pair_sm100.cu",
                                "gemm_rowpair_sm100.cu", "gemm_common.cuh", "common.cuh"],
                  "combine": ["combine.cu", "common.cuh"]}


DEFAULT_WORKLOAD = "shared64_T4096_dropless"
SIDE_WORKLOADS = ("granite24", "mixtral_prefill", "mixtral_decode", "shared64_T16_dropless",
                  "switch_phi125", "switch_phi125_reroute", "shared64_T4096_phi1_reroute")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--also", default=",".join(SIDE_WORKLOADS),
                    help="comma-separated workloads measured after the headline one, reported "
                         "under 'workloads' ('none' for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--profiled-steps", type=int, default=20,
                    help="replays of the event-instrumented graph, after the timed region, "
                         "that give the per-kernel times")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the workload's layer count (a stack of fewer layers)")
    ap.add_argument("--stats", action="store_true",
                    help="also gather routing statistics: the router's per-tile sums and one "
                         "moe_routing_stats call per layer")
    ap.add_argument("--tiles", default="auto", choices=["auto", "rows", "columns", "pairs"],
                    help="expert-FFN tile shape (bf16)")
    ap.add_argument("--fuse", default="none", choices=["none", "gather", "combine", "gather+combine"],
                    help="steps fused into the expert GEMMs (workloads with the reroute policy "
                         "or fp32 run unfused)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch through the library call by call instead of replaying a CUDA graph")
    a = ap.parse_args(argv)
    a.warmup = max(a.warmup, 3)
    a.also = [] if a.also in ("", "none") else [w for w in a.also.split(",") if w != a.workload]
    return a


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    Q = ("timestamp,index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,"
         "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id=None):
        self.proc = None
        self.bus_id = bus_id
        self.path = tempfile.mktemp(suffix=".csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv",
                                          "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self, t0, t1):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                if len(r) < 11 or r[0].startswith("timestamp"):
                    continue
                r = [c.strip() for c in r]
                try:
                    ts = time.mktime(time.strptime(r[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + r[0].split(".")[1]) if "." in r[0] else 0.0
                except ValueError:
                    continue
                rows.append((ts, r))
        os.unlink(self.path)
        if self.bus_id:
            sel = [x for x in rows if x[1][2].lower().endswith(self.bus_id.lower()[-12:])]
            rows = sel or rows
        inside = [x for x in rows if t0 - 0.1 <= x[0] <= t1 + 0.1] or rows
        if not inside:
            return None
        mhz = [float(r[3].split()[0]) for _, r in inside if r[3].split()[0].replace(".", "").isdigit()]
        mx = [float(r[4].split()[0]) for _, r in inside if r[4].split()[0].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for _, r in inside for n, v in zip(names, r[7:11]) if v == "Active"})
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(inside)}


# ----------------------------------------------------------------------------- cost model

def kernel_costs(wl, R, touched):
    """Algorithmic bytes and flops per launch of each kernel for one layer.

    R: kept routed rows; touched: experts with at least one kept row."""
    esz = 2 if wl.dtype == "bf16" else 4
    T, d, E, k, F = wl.T, wl.d, wl.E, wl.k, wl.d_ff
    sh = 1 if wl.has_shared else 0
    Rp = R + sh * T                     # rows through the expert GEMMs
    nw = touched + sh                   # weight sets streamed
    c = {}
    c["route"] = dict(bytes=T * d * esz + E * d * esz + T * k * 8 + E * 4, flops=2.0 * T * d * E)
    c["pack"] = dict(bytes=T * d * esz + R * d * esz + T * k * 8 + R * 4, flops=0.0)
    c["gemm_gate_up"] = dict(bytes=nw * 2 * F * d * esz + Rp * d * esz + Rp * F * esz,
                             flops=4.0 * Rp * d * F)
    c["gemm_down"] = dict(bytes=nw * d * F * esz + Rp * F * esz + Rp * d * esz,
                          flops=2.0 * Rp * d * F)
    c["combine"] = dict(bytes=R * d * esz + T * d * esz * (1 + int(wl.add_residual) + sh) + T * k * 8,
                        flops=0.0)
    return c


def traffic_from_profiles(kernel, workload):
    """ncu DRAM bytes per launch recorded under profiles/, if the kernel source is unchanged."""
    pdir = os.path.join(ROOT, "profiles")
    srcdir = os.path.join(ROOT, "routing_dispatch_expert_gemm_b200", "csrc")
    h = hashlib.sha1()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(srcdir, f), "rb") as fh:
            h.update(fh.read())
    sha = h.hexdigest()[:12]
    if not os.path.isdir(pdir):
        return None
    pat = re.compile(r"traffic_bytes_per_launch\s+%s@%s\s*=\s*([0-9.eE+]+)\s+sources\s+([0-9a-f]+)"
                     % (re.escape(kernel), re.escape(workload)))
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith((".md", ".txt")):
            continue
        with open(os.path.join(pdir, fn)) as f:
            for line in f:
                m = pat.search(line)
                if m and m.group(2) == sha:
                    return float(m.group(1))
    return None


def source_sha(kernel):
    srcdir = os.path.join(ROOT, "routing_dispatch_expert_gemm_b200", "csrc")
    h = hashlib.sha1()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(srcdir, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


# ----------------------------------------------------------------------------- replicas

def max_over_ranks(x, world, device="cpu"):
    """The largest value of x over all ranks: a job is as slow as its slowest rank.  Every
    rank must call it at the same point (it is a collective when world > 1)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, world, ms_per_step):
    """Whole-job throughput: every rank processes units_per_rank_step units per step (weak
    scaling, independent replicas), and a step takes ms_per_step on the slowest rank."""
    return world * units_per_rank_step / (ms_per_step / 1e3)


# ----------------------------------------------------------------------------- CPU oracle

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_tokens(wl):
    """Tokens whose expert FFN the oracle computes per layer call in a bounded sample: all of
    them for small layers; for large ones a few, so that one call stays within seconds (the
    oracle converts every expert it touches to fp64, 3 d F values each)."""
    if wl.T * wl.k * wl.d * wl.d_ff <= 4e10:
        return None
    return 4 if wl.d * wl.d_ff >= 1e8 else 32


def oracle_sample_rate(wl, x, layers, budget_s=12.0, max_layers=None, n_tokens=None, seed=0):
    """Time the oracle as it stands on a bounded sample; returns (tokens*layers/s, sample, s).

    Routing and the capacity pass always cover all T tokens; the expert FFN and combine run
    for all tokens, or for a seeded sample of ``n_tokens`` (default: ``oracle_tokens``).
    The tensors may live on the device: the oracle converts what it reads to fp64 numpy."""
    import numpy as np

    from oracle import moe_oracle as O
    C = None if wl.phi is None else O.capacity(wl.T, wl.k, wl.E, *wl.phi)
    if n_tokens is None:
        n_tokens = oracle_tokens(wl)
    toks = None
    if n_tokens is not None and n_tokens < wl.T:
        toks = np.sort(np.random.default_rng(seed).choice(wl.T, size=n_tokens, replace=False))
    t0 = time.perf_counter()
    done = 0
    xin = x
    for p in layers:
        y, _ = O.moe_layer(xin, p, wl.k, wl.gate_mode, C, add_residual=wl.add_residual, tokens=toks,
                           layout=wl.layout, overflow=wl.overflow)
        done += 1
        if wl.add_residual and toks is None:
            xin = O.round_to_bf16(y) if wl.dtype == "bf16" else y
        if time.perf_counter() - t0 > budget_s or (max_layers and done >= max_layers):
            break
    el = time.perf_counter() - t0
    ntok = wl.T if toks is None else len(toks)
    sample = (f"{done} of {len(layers)} layers x {ntok} of {wl.T} tokens "
              f"(routing and capacity over all tokens), fp64 numpy")
    return ntok * done / el, sample, el


# ----------------------------------------------------------------------------- our arm

def _dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    return world, rank, dev


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def measure_workload(a, wl, dev, world, rank, e2e=False, cpu=False):
    """Time one workload: K replays of the plain graph of its step (the timed region), then a
    separate pass of event-instrumented replays for the per-kernel times.  Every rank calls
    it with the same arguments (the barriers and max-over-ranks are collectives)."""
    import torch

    from routing_dispatch_expert_gemm_b200 import inputs as I, native as N

    L = wl.layers
    x, layers = I.make_inputs(wl, seed=a.seed + rank, device=dev)
    cap = -1 if wl.phi is None else N.moe_capacity(wl.T, wl.k, wl.E, *wl.phi)
    fuse = a.fuse if (wl.overflow == "drop" and wl.dtype == "bf16") else "none"
    tiles = a.tiles if fuse == "none" else "auto"
    cfg = N.make_config(wl.T, wl.d, wl.E, wl.k, wl.d_ff, dtype=wl.dtype, gate_mode=wl.gate_mode,
                        capacity=cap, has_shared=wl.has_shared, add_residual=wl.add_residual,
                        layout=wl.layout, overflow=wl.overflow, stats=a.stats, tiles=tiles,
                        fuse=fuse)
    ws = N.workspace(cfg, dev)
    summ = torch.zeros((L, 32), dtype=torch.uint8, device=dev)
    ybuf = [torch.empty_like(x), torch.empty_like(x)]
    demand = torch.zeros((L, wl.E), dtype=torch.int32, device=dev)
    offsets = torch.zeros((L, N.offsets_len(cfg)), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(xin, evs=None, bufs=None):
        st_ = torch.cuda.current_stream(dev)
        h = xin
        for l, p in enumerate(layers):
            y = (ybuf if bufs is None else bufs)[l % 2]
            args = (cfg, h, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"], p["w_down"],
                    p["shared_gate"], p["shared_up"], p["shared_down"], y, None, None,
                    demand[l], offsets[l])
            if evs is None:
                N.moe_forward(*args, ws, st_)
            else:
                N.moe_forward_profiled(*args, evs[l], ws, st_)
            if a.stats:
                N.moe_routing_stats(cfg, demand[l], offsets[l], 1e-2, None, None, summ[l], ws, st_)
            h = y
        return h

    # weights + activations per step vs L2: flush only when the step fits in L2
    step_bytes = sum(t.numel() * t.element_size() for p in layers for t in p.values()
                     if t is not None)
    flush = None
    if step_bytes < 256e6:
        flush = torch.empty(int(512e6) // 4, dtype=torch.int32, device=dev)

    for _ in range(a.warmup):
        step(x)
    torch.cuda.synchronize(dev)
    st = N.moe_get_device_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"{wl.name}: device status {st} after warm-up")

    nprof = max(1, min(a.profiled_steps, a.steps))
    # one interval per step; the reroute policy's kernels get their own (seven events)
    knames = (KERNELS[:2] + ["reroute"] + KERNELS[2:]) if wl.overflow == "reroute" else KERNELS
    evs = [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(knames) + 1)]
            for _ in range(L)] for _ in range(nprof)]
    for s_ in evs:  # create the handles before capture / timing
        for l_ in s_:
            for e_ in l_:
                e_.record(stream)
    torch.cuda.synchronize(dev)

    # The step as CUDA graphs: the plain graph (timed), plus one graph per instrumented
    # replay (each with its own events).  Replaying removes the host launch overhead of
    # the library calls; every kernel still launches on every replay.
    graphs = []
    g_plain = None
    cs = torch.cuda.Stream(dev)
    if a.graph:
        g_plain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_plain, stream=cs):
            step(x)
        for i in range(nprof):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cs):
                step(x, evs[i])
            graphs.append(g)
        for _ in range(2):
            g_plain.replay()
        torch.cuda.synchronize(dev)

    def plain_step():
        if a.graph:
            g_plain.replay()
        else:
            step(x)

    def profiled_step(i):
        if a.graph:
            graphs[i].replay()
        else:
            step(x, evs[i])

    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(a.steps)]
    bus = None
    try:
        pr = torch.cuda.get_device_properties(dev)
        bus = "%02X:%02X.0" % (pr.pci_bus_id, pr.pci_device_id)
    except Exception:
        pass
    clocks = ClockSampler(bus)
    clocks.start()
    torch.cuda.synchronize(dev)
    _barrier(world)
    torch.cuda.synchronize(dev)
    t0 = time.time()
    for s_i in range(a.steps):             # ---- timed region: the plain step only
        if flush is not None:
            flush.zero_()
        step_ev[s_i][0].record(stream)
        plain_step()
        step_ev[s_i][1].record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    _barrier(world)
    clk = clocks.stop(t0, t1)
    per_step = [b.elapsed_time(e) for b, e in step_ev]
    ms_total = max_over_ranks(sum(per_step), world, dev)
    ms_per_step = ms_total / a.steps
    value = job_throughput(wl.T * L, world, ms_per_step)
    st = N.moe_get_device_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"{wl.name}: device status {st} after timing")

    # ---- per-kernel times: the instrumented replays, outside the timed region
    for i in range(nprof):
        if flush is not None:
            flush.zero_()
        profiled_step(i)
    torch.cuda.synchronize(dev)
    per = {k: [] for k in knames}
    for s in range(nprof):
        for l in range(L):
            e = evs[s][l]
            for i, kname in enumerate(knames):
                per[kname].append(e[i].elapsed_time(e[i + 1]))
    avg_ms = {k: statistics.mean(v) for k, v in per.items()}
    tot_ms = {k: sum(v) for k, v in per.items()}
    dom = max(KERNELS, key=tot_ms.get)  # the kernels with an algorithmic-bytes model

    dem = demand.cpu()
    offs = offsets.cpu()
    if wl.layout == "padded":  # filled slots per expert follow the segment starts
        Rs = [int(offs[l, wl.E + 2:].sum()) for l in range(L)]
        touched = [int((offs[l, wl.E + 2:] > 0).sum()) for l in range(L)]
    else:
        Rs = [int(offs[l, wl.E]) for l in range(L)]
        touched = [int((offs[l, 1:wl.E + 1] - offs[l, :wl.E] > 0).sum()) for l in range(L)]
    costs = [kernel_costs(wl, R, tc) for R, tc in zip(Rs, touched)]
    peaks, peak_src = load_peaks()
    # Tensor peak for the clock regime actually seen: the burst figure when the SM clock
    # stayed near its maximum during the timed region, the sustained (power-capped) one
    # otherwise.
    near_max = bool(clk and clk.get("sm_mhz") and clk.get("sm_max_mhz")
                    and clk["sm_mhz"] >= 0.95 * clk["sm_max_mhz"])
    if near_max or "bf16_tflops_sustained" not in peaks:
        pk_tc, tc_kind = peaks["bf16_tflops"], "burst"
    else:
        pk_tc, tc_kind = peaks["bf16_tflops_sustained"], "sustained"
    pk_hbm = peaks["hbm_gbs"]

    def roof(kname):
        b = statistics.mean(c[kname]["bytes"] for c in costs)
        fl = statistics.mean(c[kname]["flops"] for c in costs)
        t_s = avg_ms[kname] / 1e3
        t_tc = fl / (pk_tc * 1e12)
        t_hbm = b / (pk_hbm * 1e9)
        if t_tc >= t_hbm:
            ach = fl / t_s / 1e12
            r = {"bound": "tensor", "achieved": ach, "peak": pk_tc, "unit": "TFLOP/s",
                 "frac": ach / pk_tc}
        else:
            ach = b / t_s / 1e9
            r = {"bound": "hbm", "achieved": ach, "peak": pk_hbm, "unit": "GB/s",
                 "frac": ach / pk_hbm}
        spec = SPEC_PEAKS["bf16_tflops"] if r["bound"] == "tensor" else SPEC_PEAKS["hbm_gbs"]
        r.update(spec_peak=spec, frac_of_spec=r["achieved"] / spec)
        r.update(kernel=kname, algorithmic_bytes=b, algorithmic_flops=fl,
                 avg_launch_us=avg_ms[kname] * 1e3,
                 peak_source=f"{peak_src} ({tc_kind} tensor figure)" if r["bound"] == "tensor"
                 else peak_src)
        return r

    roofline = roof(dom)
    roofline["traffic"] = traffic_from_profiles(dom, wl.name)
    roofline["source_sha"] = source_sha(dom)
    roofline["timing"] = (f"average of {nprof} event-instrumented replays after the timed "
                          f"region, on the launching stream")
    breakdown = {k: {"avg_us": round(avg_ms[k] * 1e3, 2), "share": round(tot_ms[k] / sum(tot_ms.values()), 4),
                     "frac": round(roof(k)["frac"], 4), "frac_of_spec": round(roof(k)["frac_of_spec"], 4),
                     "bound": roof(k)["bound"]} for k in KERNELS}
    if "reroute" in per:  # the placement is a latency chain: time and share only
        breakdown["reroute"] = {"avg_us": round(avg_ms["reroute"] * 1e3, 2),
                                "share": round(tot_ms["reroute"] / sum(tot_ms.values()), 4),
                                "bound": "latency"}
    launches = L * ((6 if wl.overflow == "reroute" else 3) + N.moe_ffn_launches(cfg) + int(a.stats)
                    - (1 if "combine" in fuse else 0))

    out = {"workload": wl.name, "ms_per_step": ms_per_step,
           "ffn_tiles": N.moe_ffn_tile_shape(cfg) if wl.dtype == "bf16" else "cuda-core",
           "fuse": fuse,
           "ms_per_step_median": statistics.median(per_step), "value": value, "unit": UNIT,
           "layers": L, "routes_per_step": int(dem.sum()), "kept_rows_per_step": int(sum(Rs)),
           "capacity": cap, "roofline": roofline, "kernels": breakdown, "clocks": clk,
           "launches_per_step": launches,
           "l2": ("flushed between steps" if flush is not None else
                  f"inputs larger than L2 ({step_bytes / 1e9:.2f} GB of weights per step)")}

    if e2e:
        # End to end through the public API: pinned host x in, pinned host y out, every
        # step.  With graphs the copies run on two copy streams and overlap the neighbouring
        # steps' compute (step i+1's x is uploaded while step i computes, step i's y is read
        # back while step i+1 computes), with two input buffers and two captured steps that
        # have their own output buffers; all copies are inside the timed region.
        nbytes = x.numel() * x.element_size()
        x_host = x.cpu().pin_memory()
        y_hosts = [torch.empty_like(x_host).pin_memory() for _ in range(2)]
        x_devs = [torch.empty_like(x) for _ in range(2)]
        if a.graph:
            out_bufs = [[torch.empty_like(x), torch.empty_like(x)] for _ in range(2)]
            g_e2e, outs = [], []
            for b in range(2):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cs):
                    outs.append(step(x_devs[b], bufs=out_bufs[b]))
                g_e2e.append(g)
            cp_in, cp_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            ev_in = [torch.cuda.Event() for _ in range(2)]    # x_devs[b] uploaded
            ev_comp = [torch.cuda.Event() for _ in range(2)]  # step in buffer b computed
            ev_out = [torch.cuda.Event() for _ in range(2)]   # its y read back
            ev_go = torch.cuda.Event()

            def run_e2e(k):
                ev_go.record(stream)
                cp_in.wait_event(ev_go)
                with torch.cuda.stream(cp_in):
                    x_devs[0].copy_(x_host, non_blocking=True)
                ev_in[0].record(cp_in)
                for i in range(k):
                    b = i % 2
                    if i + 1 < k:  # the next step's x, once step i-1 has read that buffer
                        if i >= 1:
                            cp_in.wait_event(ev_comp[1 - b])
                        with torch.cuda.stream(cp_in):
                            x_devs[1 - b].copy_(x_host, non_blocking=True)
                        ev_in[1 - b].record(cp_in)
                    stream.wait_event(ev_in[b])
                    if i >= 2:  # step i-2's y (same buffers) has been read back
                        stream.wait_event(ev_out[b])
                    if flush is not None:
                        flush.zero_()
                    g_e2e[b].replay()
                    ev_comp[b].record(stream)
                    cp_out.wait_event(ev_comp[b])
                    with torch.cuda.stream(cp_out):
                        y_hosts[b].copy_(outs[b], non_blocking=True)
                    ev_out[b].record(cp_out)
                stream.wait_event(ev_out[(k - 1) % 2])
                if k >= 2:
                    stream.wait_event(ev_out[k % 2])
        else:
            def run_e2e(k):
                for i in range(k):
                    x_devs[0].copy_(x_host, non_blocking=True)
                    if flush is not None:
                        flush.zero_()
                    y_hosts[i % 2].copy_(step(x_devs[0]), non_blocking=True)

        run_e2e(2)
        torch.cuda.synchronize(dev)
        _barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run_e2e(a.steps)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / a.steps
        out["e2e"] = {"value": job_throughput(wl.T * L, world, e2e_ms), "unit": UNIT,
                      "ms_per_step": e2e_ms, "h2d_bytes_per_step": nbytes,
                      "d2h_bytes_per_step": nbytes,
                      "copies": ("two copy streams overlapping the neighbouring steps' compute"
                                 if a.graph else "in order with the compute")}
        out["output_finite"] = bool(torch.isfinite(y_hosts[(a.steps - 1) % 2].float()).all().item())
        if a.graph:
            del g_e2e
    del graphs, g_plain

    if cpu:
        rate, sample, el = oracle_sample_rate(wl, x, layers)
        out["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": blas_threads(),
                               "kind": "oracle", "sample": sample, "seconds": round(el, 2)}
    del x, layers, ws, ybuf, flush
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return out


def run_ours(a):
    import torch
    import torch.distributed as dist

    from routing_dispatch_expert_gemm_b200 import build, inputs as I, native as N

    world, rank, dev = _dist_setup()
    if rank == 0:
        build.build()
    _barrier(world)
    N.lib()

    wl = I.WORKLOADS[a.workload]
    if a.layers is not None:
        wl = wl.with_(layers=a.layers)
    head = measure_workload(a, wl, dev, world, rank, e2e=True,
                            cpu=(rank == 0 and world == 1 and not a.no_cpu_baseline))
    side = {}
    for name in a.also:
        r = measure_workload(a, I.WORKLOADS[name], dev, world, rank)
        side[name] = {k: r[k] for k in ("ms_per_step", "value", "unit", "layers",
                                        "routes_per_step", "capacity", "ffn_tiles", "fuse",
                                        "kernels", "clocks", "l2")}
        rf = r["roofline"]
        side[name]["roofline"] = {k: rf[k] for k in ("kernel", "bound", "achieved", "peak", "unit",
                                                    "frac", "frac_of_spec", "traffic")}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    wl_cfg = {"workload": wl.name, "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "d_ff": wl.d_ff,
              "layers": wl.layers, "gate_mode": wl.gate_mode, "capacity": head["capacity"],
              "shared_expert": wl.has_shared, "residual": wl.add_residual, "layout": wl.layout,
              "overflow": wl.overflow, "routing_stats": a.stats,
              "parallelism": f"replicas{world}", "cuda_graph": a.graph, "l2": head["l2"],
              "ffn_tiles": head["ffn_tiles"], "fuse": head["fuse"]}
    out = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": head["ms_per_step"],
        "ms_per_step_median": head["ms_per_step_median"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": wl_cfg, "roofline": head["roofline"], "kernels": head["kernels"],
        "cpu_baseline": head.get("cpu_baseline"), "e2e": head["e2e"],
        "gpu_launches": a.steps * head["launches_per_step"], "clocks": head["clocks"],
        "routes_per_step": head["routes_per_step"], "output_finite": head["output_finite"],
        "workloads": side,
    }
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------- reference arm

def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import torch

    from routing_dispatch_expert_gemm_b200 import inputs as I

    wl = I.WORKLOADS[a.workload]
    # The inputs stay where they are drawn (the device when there is one); the oracle
    # converts what it reads to fp64 numpy on the host and computes there.
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x, layers = I.make_inputs(wl, seed=a.seed, device=dev, layers=1)
    # per step: one layer, routing over all tokens, the FFN on a seeded token sample
    nt = min(wl.T, 64)
    if wl.d * wl.d_ff >= 1e8:
        nt = 2
    elif wl.d * wl.d_ff >= 1e7:
        nt = 16
    for i in range(a.warmup):
        oracle_sample_rate(wl, x, layers, budget_s=1e9, max_layers=1, n_tokens=nt, seed=i)
    t0 = time.perf_counter()
    rates = []
    sample = ""
    for i in range(a.steps):
        r, sample, _ = oracle_sample_rate(wl, x, layers, budget_s=1e9, max_layers=1, n_tokens=nt,
                                          seed=1000 + i)
        rates.append(r)
    el = time.perf_counter() - t0
    value = statistics.mean(rates)
    cores = blas_threads()
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": el * 1e3 / a.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k,
                   "d_ff": wl.d_ff, "layers": wl.layers, "gate_mode": wl.gate_mode,
                   "layout": wl.layout, "overflow": wl.overflow},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": "per step: " + sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    a = parse_args()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
