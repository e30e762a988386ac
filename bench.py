#!/usr/bin/env python
"""Benchmark of the Muon optimizer step on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload d24] [--impl muon|reference]

A step is one muon_step over the whole parameter set (momentum + norm, k
Newton-Schulz iterations of Gram / polynomial / update, parameter write), with
W, G and M resident in HBM.  Inputs are synthetic and seeded
(muon_newton_schulz_07_b200.inputs).  Under torchrun every rank steps its own
parameter set (weak scaling) and the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Muon optimizer steps/s per param set; NS TFLOP/s & % of B200 bf16 dense peak"
UNIT = "steps/s"
# The B200 L2 holds 126 MB: inputs below twice that are flushed from it between timed steps.
L2_FLUSH_BELOW = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["muon", "reference"], default="muon")
    ap.add_argument("--workload", default="d24", choices=["single256", "gpt2s", "d24", "l38b", "stress"])
    ap.add_argument("--ns-steps", type=int, default=5)
    ap.add_argument("--mode", choices=["replica", "sharded"], default="replica",
                    help="replica: every rank steps its own parameter set (weak scaling); sharded: the ranks "
                         "split one set by matrix and all-gather the parameters (strong scaling)")
    ap.add_argument("--matrices", type=int, default=0,
                    help="use only the first N matrices of the workload (profiling captures of a smaller case)")
    ap.add_argument("--schedule", choices=["auto", "staged", "fused", "split"], default="auto",
                    help="Newton-Schulz launch schedule of the library (staged: one launch per stage)")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of CUDA graphs of the step (captured through the C ABI) instead of eager calls")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-adamw", action="store_true", help="skip the AdamW leg (non-matrix parameters)")
    ap.add_argument("--reference-budget-s", type=float, default=150.0)
    ap.add_argument("--extra", default=",".join(EXTRA_LEGS),
                    help="further workloads timed after the d24 headline on one GPU (comma list of "
                         + ", ".join(EXTRA_LEGS) + "; empty to skip)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS if k in p}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def flops_by_kind(shapes, k):
    """Algorithmic flops per step (2 per multiply-add; the symmetric products counted once)."""
    gram = poly = upd = 0
    for r, c in shapes:
        m, n = min(r, c), max(r, c)
        gram += m * m * n
        poly += m ** 3
        upd += 2 * m * m * n
    return {"gram": k * gram, "poly": k * poly, "update": k * upd}


def bytes_by_kind(shapes, elem=2):
    n = sum(r * c for r, c in shapes)
    # momentum_norm: read G, M; write M1 (elem bytes each) and the bf16 X0.
    # write: read W (elem) and the bf16 final X, write W (elem).
    return {"momentum_norm": (3 * elem + 2) * n, "write": (2 * elem + 2) * n}


def measured_traffic(kind, workload):
    """DRAM bytes (read + write) per launch of the dominant kernel from the committed ncu capture,
    scaled to the workload; None unless the capture matches this kernel source and workload."""
    import hashlib

    path = os.path.join(ROOT, "profiles", f"traffic_{kind}_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != rec["source_sha256_16"]:
            return None  # the kernel changed since the counters were taken
    scale = rec["scale_to_workload"].get(workload)
    if scale is None:
        return None
    return (rec["dram_bytes_read"] + rec["dram_bytes_write"]) * scale


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        info = [d for d in threadpool_info() if d.get("user_api") == "blas"]
        if info:
            return int(max(d.get("num_threads", 1) for d in info))
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="muon_clocks_", suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
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
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) == 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")

        sm = [num(r[1]) for r in rows]
        mx = [num(r[2]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": reasons, "samples": len(rows),
                "power_w_max": max(num(r[3]) for r in rows)}


def gpu_index_for(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ---------------------------------------------------------------- oracle timings (CPU)

def oracle_sample(wl, max_seconds=30.0):
    """Time the float64 oracle on one matrix of each distinct shape; extrapolate to the set."""
    import numpy as np

    import oracle as O
    from muon_newton_schulz_07_b200 import inputs as I

    first = {}
    for i, s in enumerate(wl.shapes):
        first.setdefault(s, i)
    counts = {s: wl.shapes.count(s) for s in first}
    hp = O.Hyper(lr=0.02, beta=0.95, weight_decay=0.0, eps=1e-7, nesterov=True, ns_steps=5)
    per_shape = {}
    t_all = time.perf_counter()
    for s, i in first.items():
        W, G, M = I.weight(wl, i).astype(np.float64), I.gradient(wl, 1, i).astype(np.float64), \
            I.momentum(wl, i).astype(np.float64)
        t0 = time.perf_counter()
        O.muon_step(W, G, M, hp)
        per_shape[s] = time.perf_counter() - t0
        if time.perf_counter() - t_all > max_seconds:
            break
    if len(per_shape) < len(first):
        # budget ran out: scale the rest by flops from the timed shapes
        rate = sum(O.ns_flops(*s, 5) for s in per_shape) / sum(per_shape.values())
        for s in first:
            per_shape.setdefault(s, O.ns_flops(*s, 5) / rate)
    step_s = sum(counts[s] * per_shape[s] for s in first)
    sample = "one matrix of each distinct shape (" + ", ".join(f"{r}x{c}" for r, c in first) + \
        f"), float64 NumPy oracle, scaled by shape counts to the {len(wl.shapes)}-matrix set (extrapolated)"
    return step_s, sample


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank):
    if rank != 0:
        return
    from muon_newton_schulz_07_b200 import inputs as I

    import numpy as np

    import oracle as O

    wl = I.WORKLOADS[args.workload]
    first = {}
    for i, s in enumerate(wl.shapes):
        first.setdefault(s, i)
    shapes = list(first)
    counts = {s: wl.shapes.count(s) for s in shapes}
    hp = O.Hyper(ns_steps=args.ns_steps)
    times = {s: [] for s in shapes}
    t_begin = time.perf_counter()
    done = 0
    # the timed steps start over at the first shape and cover every shape at least once
    n_timed = max(args.steps, len(shapes))
    for it in range(args.warmup + n_timed):
        s = shapes[(it if it < args.warmup else it - args.warmup) % len(shapes)]
        i = first[s]
        W, G, M = (I.weight(wl, i).astype(np.float64), I.gradient(wl, 1 + it, i).astype(np.float64),
                   I.momentum(wl, i).astype(np.float64))
        t0 = time.perf_counter()
        O.muon_step(W, G, M, hp)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            times[s].append(dt)
            done += 1
        if time.perf_counter() - t_begin > args.reference_budget_s and all(times[x] for x in shapes):
            break
    step_s = sum(counts[s] * statistics.median(times[s]) for s in shapes)
    value = 1.0 / step_s
    cores = blas_threads()
    sample = (f"each timed step is one matrix of one distinct shape, cycling through "
              f"{', '.join(f'{r}x{c}' for r, c in shapes)}; the full-set step time is the sum over shapes of "
              f"count x median time (extrapolated)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "ms_per_step_is_estimate": True,
        "timed": {"unit": "one single-matrix oracle step (one matrix of one distinct shape)",
                  "count": done, "per_shape_median_s": {f"{r}x{c}": statistics.median(times[(r, c)])
                                                        for r, c in shapes},
                  "full_step_estimate": "sum over shapes of matrix count x median single-matrix time"},
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "matrices": len(wl.shapes), "params": I.param_count(wl),
                   "ns_steps": args.ns_steps},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- the Muon arm

NS_KINDS = ("gram", "poly", "update", "ns_small", "ns_fused")
# Targets for the two kinds of kernel: the Newton-Schulz products at >= 60 % of the dense bf16
# tensor peak, the momentum/norm pass at >= 80 % of the HBM copy bandwidth.
TARGET_NS_FRAC = 0.60
TARGET_MOMENTUM_FRAC = 0.80


def kernel_table(prof, shapes, k, elem, steps, peaks, peak_src, wl_name):
    """Per-kernel times from the library's event tracing, turned into rates against the peaks.

    The headline fraction of a tensor-core kernel is taken against the burst bf16 peak (the
    kernels run near the maximum clock inside a step of tens of milliseconds); the fraction of the
    sustained (power-capped) peak is given beside it.
    """
    fl = flops_by_kind(shapes, k)
    by = bytes_by_kind(shapes, elem)
    kern = {kname: {"ms_total": ms, "launches": cnt, "ms_per_launch": (ms / cnt if cnt else None),
                    "ms_per_step": ms / steps}
            for kname, (ms, cnt) in prof.items() if cnt}
    # Algorithmic work of each kind per step; rates are work per step over that kind's time per
    # step, so a kind that takes several launches per step (more than 192 matrices, more than six
    # shape groups, the norm's finishing pass) is counted once.
    per_step_units = {
        "gram": fl["gram"], "poly": fl["poly"], "update": fl["update"],
        "momentum_norm": by["momentum_norm"], "write": by["write"],
        "ns_small": sum(fl.values()), "ns_fused": sum(fl.values()),
    }
    for kname, kd in kern.items():
        if kname in NS_KINDS:
            kd["tflops"] = per_step_units[kname] / (kd["ms_per_step"] * 1e-3) / 1e12
            kd["frac_of_burst_peak"] = kd["tflops"] / peaks["bf16_tflops"]
            kd["frac_of_sustained_peak"] = kd["tflops"] / peaks["bf16_tflops_sustained"]
        elif kname in ("momentum_norm", "write"):
            kd["gbs"] = per_step_units[kname] / (kd["ms_per_step"] * 1e-3) / 1e9
            kd["frac_of_hbm"] = kd["gbs"] / peaks["hbm_gbs"]
    dominant = max(kern, key=lambda x: kern[x]["ms_total"])
    if dominant in NS_KINDS:
        ach = kern[dominant]["tflops"]
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"], "traffic": measured_traffic(dominant, wl_name),
                "kernel": {"ns_small": "ns_small_kernel", "ns_fused": "ns_fused_kernel (every iteration)"}.get(
                    dominant, f"ns_gemm_tc_kernel ({dominant})"),
                "peak_source": f"{peak_src} bf16_tflops (burst, dense)",
                "frac_sustained": ach / peaks["bf16_tflops_sustained"],
                "peak_sustained": peaks["bf16_tflops_sustained"]}
    else:
        ach = kern[dominant]["gbs"]
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": None, "kernel": dominant,
                "peak_source": f"{peak_src} hbm_gbs"}
    ns_ms = sum(kern[x]["ms_total"] for x in NS_KINDS if x in kern) / steps
    ns_flops = sum(fl.values())
    ns_tflops = ns_flops / (ns_ms * 1e-3) / 1e12 if ns_ms > 0 else None
    ns = {"tflops": ns_tflops,
          "frac_of_burst_peak": (ns_tflops / peaks["bf16_tflops"]) if ns_tflops else None,
          "frac_of_sustained_peak": (ns_tflops / peaks["bf16_tflops_sustained"]) if ns_tflops else None,
          "ms_per_step": ns_ms, "flops_per_step": ns_flops}
    targets = {"ns_frac_of_burst_peak": {"value": ns["frac_of_burst_peak"], "target": TARGET_NS_FRAC,
                                         "met": bool(ns_tflops and ns["frac_of_burst_peak"] >= TARGET_NS_FRAC)}}
    if "momentum_norm" in kern:
        f = kern["momentum_norm"]["frac_of_hbm"]
        targets["momentum_norm_frac_of_hbm"] = {"value": f, "target": TARGET_MOMENTUM_FRAC,
                                                "met": bool(f >= TARGET_MOMENTUM_FRAC)}
    return kern, roof, ns, targets


def make_inputs(wl, dev, dt, rank, shapes=None):
    """W, M and two gradient sets of a workload on the device (seeded; every rank its own G)."""
    from concurrent.futures import ThreadPoolExecutor

    from muon_newton_schulz_07_b200 import inputs as I

    n = len(shapes if shapes is not None else wl.shapes)

    def to_dev(a):
        return torch_from(a, dev, dt)

    def gen(fn):
        with ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:
            return [to_dev(a) for a in ex.map(fn, range(n))]

    W = gen(lambda i: I.weight(wl, i))
    if wl.name.startswith("stress"):
        # P diag(s) Q^T drawn on the device (host QR of the whole set takes minutes); G = M
        import torch

        M = [I.stress_momentum_torch(wl, i, dev).to(dt) for i in range(n)]
        G_sets = [[m.clone() for m in M] for _ in range(2)]
        torch.cuda.synchronize(dev)
        return W, M, G_sets
    M = gen(lambda i: I.momentum(wl, i))
    G_sets = [gen(lambda i, s=s: I.gradient(wl, 1 + s + 1000 * rank, i)) for s in range(2)]
    return W, M, G_sets


def torch_from(a, dev, dt):
    import torch

    return torch.from_numpy(a).to(dev).to(dt)


def timed_steps(step_fn, G_sets, steps, warmup, op, dev, stream, local_rank, sync_all, in_bytes, B, graph=False):
    """W warm-up steps, then `steps` timed steps with CUDA events on the launching stream; clocks
    sampled meanwhile.  Inputs smaller than L2 get a 512 MB scratch write before every timed step
    (outside that step's events).

    Eager: the timed steps also carry the library's per-kernel tracing.  Graph: one step per
    gradient set is captured into a CUDA graph (the library's muon_step is capturable) and the
    timed steps replay them, which removes the host's per-launch cost and the gaps between
    launches; the per-kernel times then come from a separate traced eager pass of the same
    steps.  Returns (ms_total, per-kernel profile, clocks, flushed, eager ms per step or None).
    """
    import torch

    for i in range(warmup):
        step_fn(G_sets[i % 2])
    sync_all()
    if op.status() != B.MUON_OK:
        raise RuntimeError("device status after warm-up is not OK")
    graphs = None
    if graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        graphs = [torch.cuda.CUDAGraph() for _ in range(2)]
        with torch.cuda.stream(side):
            for i in range(2):
                with torch.cuda.graph(graphs[i], stream=side):
                    step_fn(G_sets[i])
        stream.wait_stream(side)
        for i in range(2):  # a replay of each before timing
            graphs[i].replay()
        sync_all()

    def one(i):
        if graphs is not None:
            graphs[i % 2].replay()
        else:
            step_fn(G_sets[i % 2])

    clocks = ClockSampler(gpu_index_for(local_rank))
    clocks.start()
    time.sleep(0.3)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if in_bytes < L2_FLUSH_BELOW else None
    if graphs is None:
        B.muon_profile_begin(op.handle, steps)
    sync_all()
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            one(i)
        e1.record(stream)
        sync_all()
        ms_total = e0.elapsed_time(e1)
    else:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            one(i)
            ev[i][1].record(stream)
        sync_all()
        ms_total = sum(a.elapsed_time(b) for a, b in ev)
    clk = clocks.stop()
    eager_ms = None
    if graphs is None:
        prof = B.muon_profile_end(op.handle)
    else:
        # per-kernel times from a traced eager pass (same steps, outside the timed region)
        B.muon_profile_begin(op.handle, steps)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            step_fn(G_sets[i % 2])
        e1.record(stream)
        sync_all()
        prof = B.muon_profile_end(op.handle)
        eager_ms = e0.elapsed_time(e1) / steps
        del graphs
    status = op.status()
    if status != B.MUON_OK:
        raise RuntimeError(f"device status after the timed steps: {B.STATUS.get(status, status)}")
    return ms_total, prof, clk, flush is not None, eager_ms


# Further workloads timed after the headline one (one GPU only), each its own block of the line.
# (workload, Newton-Schulz steps, timed steps): every timed region at least about half a second,
# long enough for the GPU to reach the clock its power cap holds (a 70 ms region of the GPT-2-small
# set ran before the cap had pulled the clock down) and for the clock sampler to see it.
EXTRA_LEGS = {
    "l38b": ("l38b", 5, 10),
    "stress_k5": ("stress", 5, 30),
    "stress_k10": ("stress", 10, 15),
    "gpt2s": ("gpt2s", 5, 400),
}


def ns_schedule_taken(kern):
    """How the Newton-Schulz iterations ran, from the kernels the trace saw."""
    if "ns_small" in kern:
        return "small-matrix kernel: every iteration of a matrix on chip, one launch"
    if "ns_fused" in kern:
        return "single launch: every stage of every iteration"
    return "staged: one launch per stage"


def run_extra_leg(leg, warmup, dev, local_rank, peaks, peak_src, schedule="auto", cache=None, graph=False):
    """One further workload leg; `cache` keeps the last workload's inputs for the next leg."""
    import torch

    from muon_newton_schulz_07_b200 import binding as B
    from muon_newton_schulz_07_b200 import inputs as I
    from muon_newton_schulz_07_b200.optimizer import MuonStep

    name, k, steps = EXTRA_LEGS[leg]
    wl = I.WORKLOADS[name]
    shapes = list(wl.shapes)
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    t0 = time.perf_counter()
    if cache is not None and cache.get("name") == name:
        W, M, G_sets = cache["inputs"]
    else:
        if cache is not None:
            cache.clear()
            torch.cuda.empty_cache()
        W, M, G_sets = make_inputs(wl, dev, dt, 0)
        if cache is not None:
            cache.update(name=name, inputs=(W, M, G_sets))
    gen_s = time.perf_counter() - t0
    op = MuonStep(shapes, dtype=dt, device=dev, schedule=schedule)
    stream = torch.cuda.current_stream(dev)

    def step_fn(Gs):
        op(W, Gs, M, ns_steps=k)

    in_bytes = sum(t.numel() * t.element_size() for t in list(W) + list(M) + list(G_sets[0]))
    ms_total, prof, clk, flushed, eager_ms = timed_steps(step_fn, G_sets, steps, warmup, op, dev, stream, local_rank,
                                                         lambda: torch.cuda.synchronize(dev), in_bytes, B, graph)
    kern, roof, ns, targets = kernel_table(prof, shapes, k, 4 if dt == torch.float32 else 2, steps, peaks, peak_src,
                                           wl.name)
    ms = ms_total / steps
    out = {"workload": wl.name, "ns_steps": k, "matrices": len(shapes), "params": I.param_count(wl),
           "schedule": schedule, "ns_schedule": ns_schedule_taken(kern), "steps": steps, "warmup": warmup, "ms_per_step": ms, "value": 1000.0 / ms, "unit": UNIT,
           "roofline": roof, "ns": ns, "kernels": kern, "targets": targets,
           "gpu_launches": op.launches_per_step(k) * steps, "clocks": clk,
           "l2": "flushed before every timed step" if flushed else "inputs larger than L2, no flush",
           "input_generation_s": gen_s, "launch": "cuda graph replay" if graph else "eager",
           "eager_ms_per_step": eager_ms}
    op.close()
    del W, M, G_sets
    if cache is None:
        torch.cuda.empty_cache()
    return out


def run_muon(args, rank, world, local_rank):
    import numpy as np
    import torch

    from muon_newton_schulz_07_b200 import binding as B
    from muon_newton_schulz_07_b200 import inputs as I
    from muon_newton_schulz_07_b200.optimizer import MuonStep

    dist = None
    if world > 1:
        import torch.distributed as dist

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = I.WORKLOADS[args.workload]
    if args.matrices:
        import dataclasses

        wl = dataclasses.replace(wl, shapes=wl.shapes[:args.matrices], name=f"{wl.name}[:{args.matrices}]")
    shapes = list(wl.shapes)
    n = len(shapes)
    k = args.ns_steps
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16

    # Every rank steps its own parameter set; gradients differ by rank through the step seed.
    W, M, G_sets = make_inputs(wl, dev, dt, rank, shapes)
    sharded = args.mode == "sharded" and world > 1
    if sharded:
        # strong scaling: each rank owns a share of the matrices, steps only those and all-gathers W
        from muon_newton_schulz_07_b200.sharding import ShardedMuon

        probe = ShardedMuon(shapes, rank, world, local_step=lambda *a, **kw: None, ns_steps=k)
        op = MuonStep([shapes[i] for i in probe.owned], dtype=dt, device=dev, schedule=args.schedule)
        sh = ShardedMuon(shapes, rank, world, local_step=op, ns_steps=k)
        M_owned = [M[i] for i in sh.owned]

        def step_fn(Gs):
            sh.step(W, Gs, M_owned, ns_steps=k)
    else:
        op = MuonStep(shapes, dtype=dt, device=dev, schedule=args.schedule)

        def step_fn(Gs):
            op(W, Gs, M, ns_steps=k)
    launches = op.launches_per_step(k)
    stream = torch.cuda.current_stream(dev)

    def sync_all():
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x):
        if dist is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    in_bytes = sum(t.numel() * t.element_size() for t in list(W) + list(M) + list(G_sets[0]))
    ms_total, prof, clk, flushed, eager_ms = timed_steps(step_fn, G_sets, args.steps, args.warmup, op, dev, stream,
                                                         local_rank, sync_all, in_bytes, B,
                                                         args.graph and not sharded)
    ms_per_step = max_over_ranks(ms_total / args.steps)
    value = (1 if sharded else world) * 1000.0 / ms_per_step

    # ------------------------------------------------------------ end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        G_host = [[g.cpu().pin_memory() for g in gs] for gs in G_sets]
        ksteps = max(1, min(args.steps, 20))
        norms_host = torch.empty((ksteps, n), dtype=torch.float32).pin_memory()
        h2d = sum(g.numel() * g.element_size() for g in G_host[0])
        if sharded:
            # the exchange needs every rank's G on the device before the step: copy, then step
            G_dev = [torch.empty_like(g) for g in G_sets[0]]

            def host_step(Gh):
                for d, h in zip(G_dev, Gh):
                    d.copy_(h, non_blocking=True)
                step_fn(G_dev)
        else:
            # each step's G is copied on a side stream while the previous step computes
            def host_step(Gh):
                op.step_from_host(W, Gh, M, lr=0.02, beta=0.95, ns_steps=k, stream=stream)

            host_step(G_host[1])  # untimed: allocates the two device G buffers and the copy stream
        sync_all()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        if not sharded:
            op.host_copy_stream().wait_event(f0)  # the first copy starts inside the timed region
        for i in range(ksteps):
            host_step(G_host[i % 2])
            op.norms(out=norms_host[i][:len(op.shapes)])
        f1.record(stream)
        sync_all()
        assert np.isfinite(norms_host.numpy()).all()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1) / ksteps)
        e2e = {"value": (1 if sharded else world) * 1000.0 / e2e_ms, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": 4 * len(op.shapes), "ms_per_step": e2e_ms, "steps": ksteps,
               "path": ("pinned host G -> device copy, then the sharded step" if sharded else
                        "pinned host G -> device copy on a side stream overlapping the previous step "
                        "(MuonStep.step_from_host -> C ABI muon_step), per-matrix norms -> pinned host; "
                        "W and M stay resident on the device (an optimizer's state lives there), so "
                        "they are not copied back")}

    # ------------------------------------------------------------ roofline
    peaks, peak_src = load_peaks()
    kern, roof, ns, targets = kernel_table(prof, shapes, k, 4 if dt == torch.float32 else 2, args.steps, peaks,
                                           peak_src, wl.name)

    # ------------------------------------------------------------ AdamW leg (the non-matrix half)
    adamw = None
    if not args.no_adamw and wl.name == "d24":
        from concurrent.futures import ThreadPoolExecutor

        from muon_newton_schulz_07_b200.optimizer import adamw_step

        sizes = I.D24_ADAMW_SIZES
        with ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:
            P = [torch_from(a, dev, dt) for a in ex.map(lambda i: I.adamw_param(0, i, I.TID_W, sizes[i]),
                                                        range(len(sizes)))]
            Gd = [torch_from(a, dev, dt) for a in ex.map(lambda i: I.adamw_param(1, i, I.TID_G, sizes[i]),
                                                         range(len(sizes)))]
        Ma = [torch.zeros(n_, dtype=torch.float32, device=dev) for n_ in sizes]
        Va = [torch.zeros(n_, dtype=torch.float32, device=dev) for n_ in sizes]
        for i in range(args.warmup):
            adamw_step(P, Gd, Ma, Va, i + 1, lr=3e-3, betas=(0.8, 0.95), eps=1e-10, weight_decay=0.0)
        sync_all()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(args.steps):
            adamw_step(P, Gd, Ma, Va, args.warmup + i + 1, lr=3e-3, betas=(0.8, 0.95), eps=1e-10, weight_decay=0.0)
        a1.record(stream)
        sync_all()
        a_ms = max_over_ranks(a0.elapsed_time(a1) / args.steps)
        nel = sum(sizes)
        a_bytes = nel * (2 + 2 + 2 + 8 + 8)  # p read+write, g read, m and v read+write (fp32)
        a_gbs = a_bytes / (a_ms * 1e-3) / 1e9
        adamw = {"params": nel, "ms_per_step": a_ms, "gbs": a_gbs, "frac_of_hbm": a_gbs / peaks["hbm_gbs"],
                 "bytes_per_step": a_bytes, "launches_per_step": 1,
                 "set": "d24 non-matrix parameters: 14 x 32768x1536 tables + 48 scalars, bf16, fp32 moments"}
        del P, Gd, Ma, Va

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        step_s, sample = oracle_sample(wl)
        cpu = {"value": 1.0 / step_s, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample}

    # ------------------------------------------------------------ further workloads (one GPU only)
    extra = None
    if world == 1 and args.extra and wl.name == "d24" and not args.matrices:
        op.close()
        del W, M, G_sets
        torch.cuda.empty_cache()
        extra = {}
        cache = {}
        for leg in [x for x in args.extra.split(",") if x]:
            extra[leg] = run_extra_leg(leg, args.warmup, dev, local_rank, peaks, peak_src, args.schedule, cache,
                                       args.graph)
        cache.clear()
        torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "matrices": n, "params": I.param_count(wl), "ns_steps": k,
                       "groups": op.n_groups, "schedule": args.schedule, "ns_schedule": ns_schedule_taken(kern),
                       "parallelism": (f"sharded by matrix over {world} ranks + all-gather of W (NCCL)" if sharded
                                       else f"replica x{world} (one parameter set per GPU)"),
                       "l2": ("inputs larger than L2 (W, G, M: %.2f GB per GPU), no flush" % (in_bytes / 1e9)
                              if not flushed else
                              "inputs smaller than L2 (W, G, M: %.1f MB): a 512 MB buffer is written before every "
                              "timed step, outside the step's events" % (in_bytes / 1e6)),
                       "description": wl.description},
            "roofline": roof,
            "ns": ns,
            "targets": targets,
            "kernels": kern,
            "cpu_baseline": cpu,
            "adamw": adamw,
            "e2e": e2e,
            "gpu_launches": launches * args.steps,
            "clocks": clk,
            "launch": "cuda graph replay" if (args.graph and not sharded) else "eager",
            "eager_ms_per_step": eager_ms,
        }
        if extra is not None:
            line["workloads"] = extra
        print(json.dumps(line), flush=True)
    if extra is None:
        op.close()


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        try:
            run_muon(args, rank, world, local_rank)
        finally:
            dist.destroy_process_group()
    else:
        run_muon(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
