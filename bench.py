#!/usr/bin/env python
"""Benchmark of one MoGA block (router -> grouped attention -> STGA -> mean).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one call of the library's moga_layer over one batch of synthetic
inputs already resident in HBM (the whole hot path: router, counting sort,
gather, grouped attention with gate + un-permute, STGA window attention with
the two-branch mean).  Inputs are larger than L2 (126 MB), so no flush is
needed between steps.  Multi-GPU runs (torchrun) are independent replicas:
the layer has no exchange step on one node, every rank runs its own seeded
batch, and the time is the max over ranks.

Rank 0 prints ONE JSON line.  Besides the contract keys it carries the
per-stage breakdown (CUDA events recorded by the library on its own stream),
the roofline of the dominant kernel (grouped attention: useful FLOPs
4 * sum_g n_g^2 * d_h * H over the kernel's own time), the end-to-end number
through the C ABI with pinned host buffers, and the CPU oracle baseline on a
bounded sample.  ``--impl reference`` times the oracle alone (CPU).
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MoGA layer fwd tokens/s & group-attn TFLOPS (% bf16 peak) at 187k/580k ctx"
UNIT = "tokens/s"
DEFAULT_CONFIG = "video_187k"
STGA_DIRECT_MAX = 256  # largest STGA window (tokens) the library reads in place


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p["bf16_tflops_sustained"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks
class NvmlClockSampler:
    """Clocks, power and throttle reasons sampled every 20 ms by a thread
    through NVML's read-only queries, so that even a half-second timed region
    gets a few dozen samples.  Falls back to ``ClockSampler`` (nvidia-smi)."""

    PERIOD_S = 0.02

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.rows = []
        self.thread = None
        self.fallback = None

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = nv.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = nv
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM))
            try:
                self.limit_w = nv.nvmlDeviceGetEnforcedPowerLimit(self.h) / 1000.0
            except Exception:
                self.limit_w = float("nan")
        except Exception:
            self.fallback = ClockSampler(self.device_index).__enter__()
            return self
        self.stop = threading.Event()

        def loop():
            nv = self.nv
            while not self.stop.is_set():
                try:
                    sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                    pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                    rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
                    self.rows.append((sm, pw, rs))
                except Exception:
                    pass
                self.stop.wait(self.PERIOD_S)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()
        time.sleep(0.05)
        return self

    def __exit__(self, *a):
        if self.fallback is not None:
            self.fallback.__exit__(*a)
            return
        self.stop.set()
        self.thread.join(timeout=2)
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass

    def summary(self):
        if self.fallback is not None:
            return self.fallback.summary()
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        bits = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
                "sw_power_cap": 0x4}
        pmax = max(r[1] for r in self.rows)
        load = [r for r in self.rows if r[1] >= 0.5 * pmax] or self.rows
        reasons = sorted({n for r in load for n, b in bits.items() if r[2] & b})
        out = {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": self.sm_max,
               "power_w_max": pmax, "power_limit_w": self.limit_w, "samples": len(load),
               "sampler": "nvml 20 ms", "reasons": reasons}
        if len(load) < 10:
            out["few_samples"] = True
        return out


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "enforced.power.limit")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = os.path.join("/tmp", f"moga_clocks_{os.getpid()}.csv")
        ident = str(device_index)
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            pass
        self.ident = ident

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.ident, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    lim = float(parts[9]) if len(parts) > 9 else float("nan")
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9], lim))
                except ValueError:
                    continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        pmax = max(r[2] for r in rows)
        load = [r for r in rows if r[2] >= 0.5 * pmax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": pmax, "power_limit_w": rows[-1][4], "samples": len(load), "reasons": reasons}


# ----------------------------------------------------------------------------- helpers
def _stga_flops(wl):
    if wl.window is None:
        return 0.0
    import itertools
    T, Hg, Wg = wl.grid
    wt, wh, ww = wl.window
    s = 0
    for t0, h0, w0 in itertools.product(range(0, T, wt), range(0, Hg, wh), range(0, Wg, ww)):
        n = min(wt, T - t0) * min(wh, Hg - h0) * min(ww, Wg - w0)
        s += n * n
    return 4.0 * s * wl.d_h * wl.H


def _cfg(wl, world):
    return {"workload": wl.name, "N": wl.N, "H": wl.H, "d_h": wl.d_h, "d_model": wl.d, "M": wl.M,
            "grid": "x".join(map(str, wl.grid)) if wl.grid else None,
            "stga_window": "x".join(map(str, wl.window)) if wl.window else None,
            "x": f"{wl.x_kind} {wl.x_dtype}", "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"replicas x{world}"}


def _window_sizes(wl):
    """Size of the STGA window (clipped at the grid's edges) of every token."""
    T, Hg, Wg = wl.grid
    wt, wh, ww = wl.window
    tok = np.arange(wl.N)
    t, h, w = tok // (Hg * Wg), (tok // Wg) % Hg, tok % Wg
    ext = lambda c, step, size: np.minimum(step, size - (c // step) * step)
    return ext(t, wt, T) * ext(h, wh, Hg) * ext(w, ww, Wg)


def oracle_sample_time(wl, inp_cpu, seed=0, route_rows=4096):
    """Times the CPU oracle, as it stands, on bounded pieces of the layer and
    extrapolates to all N tokens and H heads.

    - route: `route_rows` tokens (independent per token, scaled by N/route_rows);
    - counting sort: all N tokens;
    - grouped attention, one head, against the largest group: the oracle with
      1 query row (the group's float64 K/V upcast plus one row) and with 1024
      rows (two of the 512-row blocks the oracle attends at a time) gives a
      cost per group token c and per (query row, key) b; the layer costs
      H * sum_g (c n_g + b n_g^2);
    - STGA, one head: the oracle over every token of the first temporal slab
      of windows, times the number of slabs and H.
    Returns (seconds for the layer, sample description, wall seconds this
    call took).
    """
    import oracle

    wall0 = time.perf_counter()
    rng = np.random.default_rng(seed)
    N, H = wl.N, wl.H
    r0 = int(rng.integers(0, max(1, N - route_rows)))
    t = time.perf_counter()
    oracle.route(inp_cpu["x"][r0:r0 + route_rows], inp_cpu["W_r"], inp_cpu["b_r"])
    t_route = (time.perf_counter() - t) * N / min(route_rows, N)
    if "gid" not in inp_cpu:
        gid, gate, margin = oracle.route(inp_cpu["x"], inp_cpu["W_r"], inp_cpu["b_r"])
        # tokens whose top-1 / top-2 logit margin is below 1e-3: the parity
        # tests exclude them from the exact group-id check
        inp_cpu["n_margin"] = int((margin < 1e-3).sum())
    else:
        gid, gate = inp_cpu["gid"], inp_cpu["gate"]
    inp_cpu["gid"], inp_cpu["gate"] = gid, gate
    t = time.perf_counter()
    oracle.counting_sort(gid, wl.M)
    t_sort = time.perf_counter() - t
    counts = np.bincount(gid, minlength=wl.M).astype(np.float64)
    big = np.nonzero(gid == int(np.argmax(counts)))[0]
    h = [int(rng.integers(0, H))]
    qkv = (inp_cpu["q"], inp_cpu["k"], inp_cpu["v"])

    def timed(fn, *args, **kw):
        t0 = time.perf_counter()
        fn(*args, **kw)
        return time.perf_counter() - t0

    rows1 = big[:1]
    rows512 = np.sort(rng.choice(big, size=min(1024, big.size), replace=False))
    t1 = timed(oracle.group_attention, *qkv, gid, gate, wl.M, rows=rows1, heads=h)
    t512 = timed(oracle.group_attention, *qkv, gid, gate, wl.M, rows=rows512, heads=h)
    n = float(big.size)
    c = t1 / n
    b = max(t512 - t1, 0.0) / (rows512.size * n)
    t_group = H * float((c * counts + b * counts ** 2).sum())
    t_stga = 0.0
    slab = ""
    if wl.window is not None:
        T, Hg, Wg = wl.grid
        wt = wl.window[0]
        rows_s = np.arange(min(wt, T) * Hg * Wg)
        t_stga = timed(oracle.stga_attention, *qkv, *wl.grid, wl.window, rows=rows_s, heads=h)
        t_stga *= H * math.ceil(T / wt)
        slab = f"; STGA over the {rows_s.size} tokens of one temporal slab of windows, one head"
    total = t_route + t_sort + t_group + t_stga
    desc = (f"router on {min(route_rows, N)} tokens scaled to N; counting sort on all {N}; grouped attention, one "
            f"head, 1 and {rows512.size} query rows against the largest group ({big.size} tokens){slab}; scaled to "
            f"all groups, windows and {H} heads (extrapolated)")
    return total, desc, time.perf_counter() - wall0


def _recorded_traffic(name):
    """DRAM bytes per grouped-attention launch from a committed ncu summary,
    or None when none was recorded for this workload or the kernel source has
    changed since the counters were taken."""
    import glob
    import hashlib
    import re

    with open(os.path.join(ROOT, "learned_token_group_b200", "csrc", "attn.cu"), "rb") as f:
        src = hashlib.sha256(f.read()).hexdigest()[:16]
    pat = re.compile(r"group_attn_traffic_bytes_per_launch\[(\w+)\] = (\d+) \(attn\.cu ([0-9a-f]+)\)")
    for fn in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(fn) as f:
            for line in f:
                m = pat.search(line)
                if m and m.group(1) == name and m.group(3) == src:
                    return int(m.group(2))
    return None


def _shot_split(T: int):
    """A fixed, uneven split of T latent frames into shots (fractions of a
    120-frame video cut at frames 24, 40, 60, 88 and 100)."""
    cuts = sorted({int(round(T * f)) for f in (0.2, 1 / 3, 0.5, 11 / 15, 5 / 6)} - {0, T})
    return [0] + cuts + [T]


def _shot_flops(wl, window, shots, aug_prev, aug_next):
    """Useful FLOPs 4 * sum over windows of q_len * kv_len * d_h * H
    (window geometry only: frames x tile area, per shot)."""
    T, Hg, Wg = wl.grid
    wt, wh, ww = window
    total = 0
    for j in range(len(shots) - 1):
        a, b = shots[j], shots[j + 1]
        step = wt if wt > 0 else b - a
        for t0 in range(a, b, step):
            t1 = min(b, t0 + step)
            extra = 0
            if t0 == a and j > 0:
                extra += a - max(shots[j - 1], a - aug_prev)
            if t1 == b and j + 1 < len(shots) - 1:
                extra += min(shots[j + 2], b + aug_next) - b
            for h0 in range(0, Hg, wh):
                for w0 in range(0, Wg, ww):
                    area = (min(Hg, h0 + wh) - h0) * (min(Wg, w0 + ww) - w0)
                    total += (t1 - t0) * area * (t1 - t0 + extra) * area
    return 4.0 * total * wl.d_h * wl.H


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


# ----------------------------------------------------------------------------- arms
def run_reference(args, wl, rank, world):
    """The oracle (CPU) as the reference arm: each step is a bounded sample."""
    if rank != 0:
        return
    inp = make_inputs(wl, seed=args.seed, device="cpu")
    desc = ""
    for _ in range(args.warmup):
        _, desc, _ = oracle_sample_time(wl, inp, seed=args.seed)
    times, walls = [], []
    for i in range(args.steps):
        t_i, desc, w_i = oracle_sample_time(wl, inp, seed=args.seed + 1 + i)
        times.append(t_i)
        walls.append(w_i)
    t = statistics.mean(times)
    value = wl.N / t
    cores = _blas_threads()
    # a step is one bounded sample: ms_per_step is its measured wall time;
    # the layer time the samples extrapolate to is reported beside it
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(walls) * 1e3,
            "layer_ms_extrapolated": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, CPU)",
            "config": _cfg(wl, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cpu_model": _cpu_model(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def max_over_ranks(value: float, dist, device=None) -> float:
    """The slowest rank's time (every rank must call this, in the same order)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measure_context(moga, wl, steps, seed, dev, dist):
    """One more workload of the metric: layer time over `steps` steps (device
    events, max over ranks), then one pass with per-stage events, reduced to
    grouped-attention TFLOP/s and router / gather bandwidth."""
    inp = make_inputs(wl, seed=seed, device=dev)
    xdt = torch.float32 if wl.x_dtype == "f32" else torch.bfloat16
    layer = moga.MogaLayer(wl.N, wl.d, wl.H, wl.d_h, wl.M, wl.grid, wl.window, xdt, dev)
    step = lambda: layer(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"])
    step()
    moga.sync_status(layer.ws)
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / steps, dist, dev)
    stages = list(moga.STAGES)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in stages]
    for b_ev, e_ev in evs:
        b_ev.record(stream)
        e_ev.record(stream)
    torch.cuda.synchronize()
    for s_i, name in enumerate(stages):
        moga.set_timing_events(name, *evs[s_i])
    step()
    for name in stages:
        moga.set_timing_events(name, None, None)
    torch.cuda.synchronize()
    moga.sync_status(layer.ws)
    st = {name: evs[s_i][0].elapsed_time(evs[s_i][1]) for s_i, name in enumerate(stages)}
    counts = np.diff(layer.offsets.cpu().numpy().astype(np.int64))
    flops = 4.0 * float((counts.astype(np.float64) ** 2).sum()) * wl.d_h * wl.H
    peaks = _peaks()
    tf = flops / (st["group_attn"] * 1e-3) / 1e12
    xb = wl.N * wl.d * (2 if wl.x_dtype == "bf16" else 4) + 8 * wl.N
    gb = 6 * wl.N * wl.H * wl.d_h * 2 + 4 * wl.N
    # A step of more than 100 ms runs the tensor cores long enough for the
    # power cap to settle the clocks, so the sustained figure is the peak of
    # such a step; the burst fraction is reported beside it.
    long_step = ms > 100.0
    peak = peaks["bf16_tflops_sustained"] if long_step else peaks["bf16_tflops"]
    out = {"workload": wl.describe(), "steps": steps, "ms_per_step": ms, "tokens_per_s": wl.N / (ms * 1e-3),
           "stage_ms": st, "group_attn_tflops": tf, "group_attn_frac_of_peak": tf / peak,
           "group_attn_peak_kind": "bf16 dense sustained (measured; step > 100 ms)" if long_step
           else "bf16 dense burst (measured)",
           "group_attn_frac_of_burst": tf / peaks["bf16_tflops"],
           "group_attn_frac_of_sustained": tf / peaks["bf16_tflops_sustained"],
           "router_GBs": xb / (st["router"] * 1e-3) / 1e9, "gather_GBs": gb / (st["gather"] * 1e-3) / 1e9,
           "largest_group": int(counts.max()), "nonempty_groups": int((counts > 0).sum())}
    if wl.window is not None:
        out["stga_attn_GBs"] = 5 * wl.N * wl.H * wl.d_h * 2 / (st["stga_attn"] * 1e-3) / 1e9
        out["stga_attn_frac_of_hbm"] = out["stga_attn_GBs"] / peaks["hbm_gbs"]
    out["router_frac_of_hbm"] = out["router_GBs"] / peaks["hbm_gbs"]
    out["gather_frac_of_hbm"] = out["gather_GBs"] / peaks["hbm_gbs"]
    del layer, inp
    return out


def run_ours(args, wl, rank, world, dist):
    import learned_token_group_b200 as moga

    dev = torch.device("cuda", torch.cuda.current_device())
    inp = make_inputs(wl, seed=args.seed + rank, device=dev)
    layer = moga.MogaLayer(wl.N, wl.d, wl.H, wl.d_h, wl.M, wl.grid, wl.window,
                           torch.float32 if wl.x_dtype == "f32" else torch.bfloat16, dev)
    step = lambda: layer(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"])

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    moga.sync_status(layer.ws)
    counts = np.diff(layer.offsets.cpu().numpy().astype(np.int64))
    flops_group = 4.0 * float((counts.astype(np.float64) ** 2).sum()) * wl.d_h * wl.H
    flops_stga = _stga_flops(wl)

    # ---- timed region: K layer steps, device time, max over ranks
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with NvmlClockSampler(dev.index) as clk:
        torch.cuda.synchronize()
        barrier()
        l0 = moga.kernel_launches()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        launches = moga.kernel_launches() - l0
    moga.sync_status(layer.ws)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dist, dev)
    clocks = clk.summary()
    if args.lean:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": wl.N * world / (ms * 1e-3), "unit": UNIT,
                              "n_gpus": world, "ms_per_step": ms, "config": _cfg(wl, world), "lean": True,
                              "gpu_launches": int(launches), "clocks": clocks}), flush=True)
        return

    # ---- per-stage breakdown: events recorded by the library around each stage
    stages = list(moga.STAGES)
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in stages]
           for _ in range(args.steps)]
    for row in evs:                      # create the CUDA events before handing them to the library
        for b_ev, e_ev in row:
            b_ev.record(stream)
            e_ev.record(stream)
    torch.cuda.synchronize()
    for i in range(args.steps):
        for s, name in enumerate(stages):
            moga.set_timing_events(name, *evs[i][s])
        step()
    for name in stages:
        moga.set_timing_events(name, None, None)
    torch.cuda.synchronize()
    stage_ms = {name: statistics.mean(evs[i][s][0].elapsed_time(evs[i][s][1]) for i in range(args.steps))
                for s, name in enumerate(stages)}

    # ---- end to end through the C ABI: pinned host inputs in, the block's
    # output back to pinned host memory, every step.  The host pipeline
    # (moga_pipe_*) overlaps a step's copies with its neighbours' compute; the
    # serial variant (copy in, compute, copy out, one after another, through
    # moga_layer on the current stream) is reported beside it for context.
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in inp.items()}
    outs_host = [torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = outs_host[0].numel() * outs_host[0].element_size()
    pipe = moga.Pipeline(wl.N, wl.d, wl.H, wl.d_h, wl.M, wl.grid, wl.window,
                         torch.float32 if wl.x_dtype == "f32" else torch.bfloat16, dev)

    def pipe_submit(i):
        pipe.submit(host["x"], host["W_r"], host["b_r"], host["q"], host["k"], host["v"], outs_host[i % 2])

    for i in range(2):
        pipe_submit(i)
    pipe.sync()
    barrier()
    n_e2e = max(3, min(args.steps, 10))
    t0 = time.perf_counter()
    for i in range(n_e2e):
        pipe_submit(i)
    pipe.sync()
    e2e_ms = max_over_ranks((time.perf_counter() - t0) * 1e3 / n_e2e, dist, dev)
    barrier()
    pipe.close()

    dinp = {k: (torch.empty_like(v) if v is not None else None) for k, v in inp.items()}

    def serial_step():
        for k, v in host.items():
            if v is not None:
                dinp[k].copy_(v, non_blocking=True)
        layer(dinp["x"], dinp["W_r"], dinp["b_r"], dinp["q"], dinp["k"], dinp["v"])
        outs_host[0].copy_(layer.out, non_blocking=True)

    serial_step()
    torch.cuda.synchronize()
    barrier()
    ev0.record(stream)
    n_serial = max(1, min(args.steps, 5))
    for _ in range(n_serial):
        serial_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    serial_ms = max_over_ranks(ev0.elapsed_time(ev1) / n_serial, dist, dev)
    del dinp
    moga.sync_status(layer.ws)

    # ---- the widened rows: three-branch block (adds the per-frame branch) and
    # routing with balancing statistics, each timed over K steps
    widened = {}
    if wl.window is not None and not args.no_extras:
        layer3 = moga.MogaLayer(wl.N, wl.d, wl.H, wl.d_h, wl.M, wl.grid, wl.window,
                                torch.float32 if wl.x_dtype == "f32" else torch.bfloat16, dev, per_frame=True)
        step3 = lambda: layer3(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"])
        step3()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            step3()
        ev1.record(stream)
        torch.cuda.synchronize()
        moga.sync_status(layer3.ws)
        widened["three_branch_layer_ms"] = ev0.elapsed_time(ev1) / args.steps
        del layer3
        # the per-frame branch alone (whole-frame windows, read in place),
        # added into an output as the block does
        frame = (1, wl.grid[1], wl.grid[2])
        ws_f = moga.workspace(moga.get_lib().stga_window_attn_workspace_size(
            wl.grid[0], wl.grid[1], wl.grid[2], moga._int3(frame), wl.H, wl.d_h), dev)
        out_f = moga.stga_window_attn(inp["q"], inp["k"], inp["v"], wl.grid, frame, ws=ws_f)
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            moga.stga_window_attn(inp["q"], inp["k"], inp["v"], wl.grid, frame, accumulate=True, out=out_f,
                                  ws=ws_f)
        ev1.record(stream)
        torch.cuda.synchronize()
        ms_f = ev0.elapsed_time(ev1) / args.steps
        L = wl.grid[1] * wl.grid[2]
        widened["per_frame_branch_ms"] = ms_f
        widened["per_frame_branch_tflops"] = 4.0 * wl.grid[0] * L * L * wl.H * wl.d_h / (ms_f * 1e-3) / 1e12
        moga.sync_status(ws_f)
        del out_f, ws_f
        # training: the forward that keeps the log-sum-exp, then the backward
        # pass (gradients of q, k, v, x, W_r, b_r) of the same block
        gen_t = torch.Generator(device=dev)
        gen_t.manual_seed(args.seed + 99)
        dout = torch.randn((wl.N, wl.H, wl.d_h), generator=gen_t, device=dev).to(torch.bfloat16)
        targs = (inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M, wl.grid, wl.window)
        tr = moga.layer_train(*targs)
        gr = moga.layer_backward(dout, tr, *targs)
        torch.cuda.synchronize()
        ev2 = torch.cuda.Event(enable_timing=True)
        t_fwd = t_bwd = 0.0
        for _ in range(args.steps):
            ev0.record(stream)
            moga.layer_train(*targs, res=tr)
            ev1.record(stream)
            moga.layer_backward(dout, tr, *targs, grads=gr)
            ev2.record(stream)
            torch.cuda.synchronize()
            t_fwd += ev0.elapsed_time(ev1)
            t_bwd += ev1.elapsed_time(ev2)
        moga.sync_status(tr["ws"])
        moga.sync_status(gr["ws"])
        t_fwd /= args.steps
        t_bwd /= args.steps
        widened["train_forward_ms"] = t_fwd
        widened["train_backward_ms"] = t_bwd
        # algorithmic backward work: five n x n x d_h products per head and
        # token set (S recomputed, dP, dV, dK, dQ) = 2.5 x the forward's
        widened["train_backward_attn_tflops"] = 2.5 * (flops_group + flops_stga) / (t_bwd * 1e-3) / 1e12
        widened["train_step_tokens_per_s"] = wl.N / ((t_fwd + t_bwd) * 1e-3)
        del tr, gr, dout
        rt = lambda: moga.route(inp["x"], inp["W_r"], inp["b_r"], wl.M, out=r_out, ws=r_ws)
        rs = lambda: moga.route_stats(inp["x"], inp["W_r"], inp["b_r"], wl.M)
        r_out = moga.route(inp["x"], inp["W_r"], inp["b_r"], wl.M)
        r_ws = moga.workspace(moga.get_lib().moga_route_workspace_size(wl.N, wl.M), dev)
        for name, fn in (("route_ms", rt), ("route_with_balance_stats_ms", rs)):
            fn()
            torch.cuda.synchronize()
            ev0.record(stream)
            for _ in range(args.steps):
                fn()
            ev1.record(stream)
            torch.cuda.synchronize()
            widened[name] = ev0.elapsed_time(ev1) / args.steps
        # shot-aware STGA over a fixed split of the latent frames into shots:
        # the pages' 2x2 spatial partition with whole-shot temporal groups, and
        # the workload's window inside shots; two boundary frames each way
        shots = _shot_split(wl.grid[0])
        ss = torch.tensor(shots, dtype=torch.int32, device=dev)
        half = (0, (wl.grid[1] + 1) // 2, (wl.grid[2] + 1) // 2)
        for tag, win in (("shot_stga_2x2_whole_shot", half), ("shot_stga_window", tuple(wl.window))):
            out_s, ws_s = moga.stga_shot_attn(inp["q"], inp["k"], inp["v"], wl.grid, win, ss, 2, 2)
            torch.cuda.synchronize()
            ev0.record(stream)
            for _ in range(args.steps):
                moga.stga_shot_attn(inp["q"], inp["k"], inp["v"], wl.grid, win, ss, 2, 2, out=out_s, ws=ws_s)
            ev1.record(stream)
            torch.cuda.synchronize()
            moga.sync_status(ws_s)
            ms_s = ev0.elapsed_time(ev1) / args.steps
            widened[tag + "_ms"] = ms_s
            widened[tag + "_tflops"] = _shot_flops(wl, win, shots, 2, 2) / (ms_s * 1e-3) / 1e12
            del out_s, ws_s
        widened["shot_split"] = shots
        # the pages' whole block in one call: MoGA, whole-shot 2x2 STGA and
        # per-frame attention, averaged (moga_layer_shots)
        blk = moga.moga_layer_shots(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M,
                                    wl.grid, half, ss, 2, 2, per_frame=True)
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            moga.moga_layer_shots(inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M, wl.grid,
                                  half, ss, 2, 2, per_frame=True, res=blk)
        ev1.record(stream)
        torch.cuda.synchronize()
        moga.sync_status(blk["ws"])
        widened["pages_block_ms"] = ev0.elapsed_time(ev1) / args.steps
        widened["pages_block"] = "MoGA + shot-aware STGA (whole shots, 2x2 tiles, 2+2 boundary frames) + per-frame"
        del blk
    # ---- variance: the same timed layer on the inputs of two more seeds
    seeds = [{"seed": args.seed, "ms_per_step": ms, "tokens_per_s": wl.N / (ms * 1e-3)}]
    if not args.no_extras:
        for extra in (1, 2):
            new = make_inputs(wl, seed=args.seed + extra + rank, device=dev)
            step_s = lambda: layer(new["x"], new["W_r"], new["b_r"], new["q"], new["k"], new["v"])
            step_s()
            torch.cuda.synchronize()
            barrier()
            ev0.record(stream)
            for _ in range(args.steps):
                step_s()
            ev1.record(stream)
            torch.cuda.synchronize()
            barrier()
            ms_s = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dist, dev)
            seeds.append({"seed": args.seed + extra, "ms_per_step": ms_s, "tokens_per_s": wl.N / (ms_s * 1e-3)})
            moga.sync_status(layer.ws)
            del new, step_s
        torch.cuda.empty_cache()
    # ---- the other contexts the metric names: the same block at 580k tokens
    # (40 heads, M = 32) and the skewed-routing stress case
    contexts = {}
    if wl.name == DEFAULT_CONFIG and not args.no_extras:
        for name, steps in (("minute_580k", 2), ("skew_187k", 5)):
            contexts[name] = measure_context(moga, WORKLOADS[name], steps, args.seed + rank, dev, dist)
            torch.cuda.empty_cache()
    if rank != 0:
        return
    peaks = _peaks()
    # The layer's clocks stay at max without power capping (sampled above), so
    # the burst figure is the denominator; the sustained one is reported beside.
    peak = peaks["bf16_tflops"]
    t_attn = stage_ms["group_attn"] * 1e-3
    attn_tflops = flops_group / t_attn / 1e12
    cpu = None
    n_margin = None
    if world == 1 and not args.no_cpu_baseline:
        cpu_inp = {k: (v.cpu() if v is not None else None) for k, v in inp.items()}
        # host timings spread by 2-3x between calls: the median of three
        est = [oracle_sample_time(wl, cpu_inp, seed=args.seed + i, route_rows=16384) for i in range(3)]
        t_cpu = statistics.median(e[0] for e in est)
        desc = est[0][1] + "; median of 3 samples"
        cpu = {"value": wl.N / t_cpu, "unit": UNIT, "cores": _blas_threads(), "cpu_model": _cpu_model(),
               "kind": "oracle", "sample": desc}
        n_margin = cpu_inp.get("n_margin")
    traffic = _recorded_traffic(wl.name)
    hbm = peaks["hbm_gbs"]
    Dbytes = wl.N * wl.H * wl.d_h * 2
    bw = {
        "router_GBs": (wl.N * wl.d * (2 if wl.x_dtype == "bf16" else 4) + 8 * wl.N) / (stage_ms["router"] * 1e-3) / 1e9,
        "gather_GBs": (6 * Dbytes + 4 * wl.N) / (stage_ms["gather"] * 1e-3) / 1e9,
        # Windows of up to 256 tokens are read in place (no gathered copy), so
        # the STGA preparation is then only the 8N-byte window permutation.
        "stga_prep_GBs": ((8 * wl.N if math.prod(wl.window) <= STGA_DIRECT_MAX else 6 * Dbytes + 8 * wl.N)
                          / (stage_ms["stga_prep"] * 1e-3) / 1e9) if wl.window else None,
        # STGA attention (HBM-bound): q, k, v read once, out read and written
        # once by the read-add epilogue
        "stga_attn_GBs": (5 * Dbytes / (stage_ms["stga_attn"] * 1e-3) / 1e9) if wl.window else None,
    }
    bw["frac_of_hbm"] = {k[:-4]: v / hbm for k, v in bw.items() if v is not None}
    line = {
        "metric": METRIC, "value": wl.N * world / (ms * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random router weights, clustered tokens)",
        "config": _cfg(wl, world),
        "group_attn_tflops": attn_tflops,
        "group_attn_frac_of_peak": attn_tflops / peak,
        "flops_vs_full_attention": (flops_group + flops_stga) / (4.0 * wl.N * wl.N * wl.d_h * wl.H),
        "stage_ms": stage_ms,
        "stage_hbm_GBs": bw,
        "group_sizes": counts.tolist(),
        "roofline": {"kernel": "attn_kernel<128> (grouped attention)", "bound": "tensor",
                     "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s", "frac": attn_tflops / peak,
                     "peak_kind": f"bf16 dense burst ({peaks['source']})",
                     "frac_of_sustained": attn_tflops / peaks["bf16_tflops_sustained"], "traffic": traffic},
        "cpu_baseline": cpu,
        "e2e": {"value": wl.N * world / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": n_e2e,
                "api": "moga_pipe_submit (host buffers; copies overlap neighbouring steps)",
                "serial": {"value": wl.N * world / (serial_ms * 1e-3), "ms_per_step": serial_ms,
                           "api": "H2D copies + moga_layer + D2H copy, one after another"}},
        "gpu_launches": int(launches),
        "clocks": clocks,
        # caller-allocated scratch of the block (the pages describe MoGA as
        # needing no additional memory beyond the permuted Q/K/V segments)
        "workspace_bytes": int(layer.ws.numel()),
        "workspace_vs_qkv": layer.ws.numel() / (3.0 * Dbytes),
        "n_margin_excluded": n_margin,
        "seeds": seeds,
        "widened": widened,
        "contexts": contexts,
    }
    print(json.dumps(line), flush=True)


def run_train(args, wl, rank, world, dist):
    """--train: the training step of the block (moga_layer_train, then
    moga_layer_backward with a seeded dout) as the timed step; one JSON line
    with the forward and backward device times.  For hardware-counter
    captures of the training kernels and for training throughput."""
    import learned_token_group_b200 as moga

    dev = torch.device("cuda", torch.cuda.current_device())
    inp = make_inputs(wl, seed=args.seed + rank, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed + 99 + rank)
    dout = torch.randn((wl.N, wl.H, wl.d_h), generator=gen, device=dev).to(torch.bfloat16)
    targs = (inp["x"], inp["W_r"], inp["b_r"], inp["q"], inp["k"], inp["v"], wl.M, wl.grid, wl.window)
    tr = moga.layer_train(*targs)
    gr = moga.layer_backward(dout, tr, *targs)
    for _ in range(max(args.warmup - 1, 0)):
        moga.layer_train(*targs, res=tr)
        moga.layer_backward(dout, tr, *targs, grads=gr)
    moga.sync_status(gr["ws"])
    counts = np.diff(tr["offsets"].cpu().numpy().astype(np.int64))
    flops = 4.0 * float((counts.astype(np.float64) ** 2).sum()) * wl.d_h * wl.H + _stga_flops(wl)
    stream = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    t_fwd = t_bwd = 0.0
    with NvmlClockSampler(dev.index) as clk:
        for _ in range(args.steps):
            if dist is not None:
                dist.barrier()
            torch.cuda.synchronize()
            ev[0].record(stream)
            moga.layer_train(*targs, res=tr)
            ev[1].record(stream)
            moga.layer_backward(dout, tr, *targs, grads=gr)
            ev[2].record(stream)
            torch.cuda.synchronize()
            t_fwd += ev[0].elapsed_time(ev[1])
            t_bwd += ev[1].elapsed_time(ev[2])
    moga.sync_status(gr["ws"])
    t_fwd = max_over_ranks(t_fwd / args.steps, dist, dev)
    t_bwd = max_over_ranks(t_bwd / args.steps, dist, dev)
    if rank == 0:
        print(json.dumps({"metric": "MoGA layer training step (forward + backward) tokens/s",
                          "value": wl.N * world / ((t_fwd + t_bwd) * 1e-3), "unit": "tokens/s", "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_fwd + t_bwd,
                          "train_forward_ms": t_fwd, "train_backward_ms": t_bwd,
                          "backward_attn_tflops": 2.5 * flops / (t_bwd * 1e-3) / 1e12,
                          "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                          "config": _cfg(wl, world), "clocks": clk.summary()}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the widened-row timings")
    ap.add_argument("--lean", action="store_true",
                    help="warm-up and timed steps only (for hardware-counter captures)")
    ap.add_argument("--train", action="store_true",
                    help="time the training step (forward keeping the log-sum-exp, then the backward pass)")
    args = ap.parse_args()
    wl = WORKLOADS[args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    dist = None
    if world > 1:
        import torch.distributed as dist_mod

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = dist_mod
    try:
        if args.train:
            run_train(args, wl, rank, world, dist)
        else:
            run_ours(args, wl, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
