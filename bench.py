#!/usr/bin/env python
"""Benchmark of the AReA attention hot path on B200 (libarea, sm_100a).

One step = one AReA attention schedule on one synthetic FLUX.1-shaped
6144x6144 image (384x384 tokens, 24 heads, head_dim 128, bf16):
  8 Phase I calls   (area_pool_kv + area_coarse_attn, f = 6 -> 64x64 keys), and
  8 Phase II calls  (area_dwt_window_plan: detail map + plan in one launch, then
                     area_window_attn; one per window side of the schedule
                     192 -> 64).
The metric is algorithmic attention TFLOP/s: 4*D*H*(query, key) pairs the
method defines (N*Nk per Phase I call; sum over windows of |W|*(|ext|+G_W)
per Phase II call) divided by the step time.  Full attention over the same
inputs is timed after the step to give the speedup ratio.

Launch: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl area|reference]
For N > 1 use torchrun; every rank runs an independent replica (the path has
no exchange step), and the job value is the sum of the ranks' work over the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "AReA attention TFLOP/s per schedule step (bf16, 1 B200)"
# Bumped whenever attn_tc.cu changes, so that stale DRAM counters are not reported.
KERNEL_REVISION = "attn_tc v14 (v13 plus a 384-thread window kernel whose warpgroups split the registers 136 / 184 with setmaxnreg)"
DEFAULT_CONFIG = "flux6144"
PUBLISHED_BF16_TFLOPS = 2250.0   # B200 dense bf16 tensor rate, published (no sparsity)


# ---------------------------------------------------------------------------
# algorithmic work (host arithmetic on plan sizes; no kernel logic here)
# ---------------------------------------------------------------------------

def phase1_flops(cfg) -> float:
    return 4.0 * cfg.B * cfg.H * cfg.N * cfg.Nk * cfg.D


def full_flops(cfg) -> float:
    return 4.0 * cfg.B * cfg.H * cfg.N * cfg.N * cfg.D


def window_flops(plan: dict, H: int, D: int) -> float:
    """4*D*H*sum_W |W|*(|ext W| + G_W) from a decoded device plan."""
    tot = 0.0
    for b in range(plan["B"]):
        nw = int(plan["nwin"][b])
        win = plan["win"][b, :nw].astype(np.float64)
        ext = plan["ext"][b, :nw].astype(np.float64)
        g = plan["gcount"][b, :nw].astype(np.float64)
        tot += float(np.sum(win[:, 2] * win[:, 3] * (ext[:, 2] * ext[:, 3] + g)))
    return 4.0 * D * H * tot


def pool_bytes(cfg) -> float:
    e = 2 if cfg.dtype == "bf16" else 4
    return 2.0 * cfg.B * cfg.H * (cfg.N + cfg.Nk) * cfg.D * e


def dwt_bytes(cfg) -> float:
    e = 2 if cfg.dtype == "bf16" else 4
    return cfg.B * cfg.N * cfg.C * e + cfg.B * (cfg.N // 4) * 4


def plan_launches(B: int) -> int:
    # the separate planner calls: header, base scores, windows, (sort init +
    # 4 x (hist, scan, scatter)) per batch element, global-KV selection,
    # weight sums
    return 5 + 13 * B


# kernels of one area_window_attn call on the tensor-core path with the
# staging area in the workspace: the copy of the windows' global-KV rows, then
# the attention kernel (the merge runs inside it); a 256-byte memset of the
# workspace counters precedes both
WINDOW_LAUNCHES = 2


# ---------------------------------------------------------------------------
# distributed plumbing (replicas; no data-path collective)
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def head_range(rank: int, world: int, H: int):
    """Contiguous heads [h0, h1) of a rank when the heads are sharded: the
    attention of each head is independent and the plan depends only on the
    detail source, so sharding needs no exchange step."""
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    return dist


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device])
        else:
            dist.barrier()


def reduce_max(dist, value: float, device: str = "cpu") -> float:
    """Max of a float over ranks (identity without a process group)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(dist, value: float, device: str = "cpu") -> float:
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path: str = ""):
        self.gpu = gpu_index
        self.proc = None
        self.path = path or os.path.join(tempfile.gettempdir(),
                                         f"area_bench_clocks_{gpu_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self) -> dict:
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons)}
        loaded = [x for x in sm if x > 0.5 * (smax or max(sm))] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the GPU workload
# ---------------------------------------------------------------------------

class AreaStep:
    """Device buffers and the call sequence of one schedule step."""

    def __init__(self, cfg, q, k, v, src, stream):
        import torch

        import step_adaptive_sparse_b200 as area
        self.area, self.torch, self.cfg, self.stream = area, torch, cfg, stream
        self.q, self.k, self.v, self.src = q, k, v, src
        dev = q.device
        self.dt = area.AREA_DTYPE_BF16 if cfg.dtype == "bf16" else area.AREA_DTYPE_F32
        self.kp = torch.empty((cfg.B, cfg.H, cfg.Nk, cfg.D), dtype=q.dtype, device=dev)
        self.vp = torch.empty_like(self.kp)
        self.o1 = torch.empty_like(q)
        self.o2 = torch.empty_like(q)
        self.energy = torch.empty((cfg.B, cfg.Hg // 2, cfg.Wg // 2), dtype=torch.float32,
                                  device=dev)
        self.pcfg, self.plan, self.plan_bytes = [], [], []
        wsb = 0
        for w in cfg.schedule:
            pc = area.make_cfg(cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
            nb = area.area_window_plan_bytes(pc)
            self.pcfg.append(pc)
            self.plan.append(torch.empty(nb, dtype=torch.uint8, device=dev))
            self.plan_bytes.append(nb)
            # the minimum plus the staging area of the global-KV rows (fast path)
            wsb = max(wsb, area.area_window_attn_ws_bytes(pc, cfg.H, cfg.D)
                      + area.area_window_attn_stage_bytes(pc, cfg.H, cfg.D))
        self.ws = torch.empty(wsb // 4, dtype=torch.float32, device=dev)
        self.ws_bytes = wsb
        self.n_phase1 = len(cfg.schedule)
        # libarea kernels per step: pool + coarse per Phase I call; the one
        # planner launch and the window call's launches per Phase II call
        self.launches = self.n_phase1 * 2 + len(cfg.schedule) * (1 + WINDOW_LAUNCHES)
        self.calls = {"pool_kv": [], "coarse_attn": [], "dwt_window_plan": [], "window_attn": []}
        self.record = False

    def _ev(self):
        return self.torch.cuda.Event(enable_timing=True)

    def _timed(self, name, fn):
        if not self.record:
            fn()
            return
        a, b = self._ev(), self._ev()
        a.record(self.stream)
        fn()
        b.record(self.stream)
        self.calls[name].append((a, b))

    def run(self):
        area, cfg, s = self.area, self.cfg, self.stream
        for _ in range(self.n_phase1):
            self._timed("pool_kv", lambda: area.area_pool_kv(
                self.k, self.v, self.kp, self.vp, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, cfg.f,
                area.AREA_POOL_MEAN, self.dt, s))
            self._timed("coarse_attn", lambda: area.area_coarse_attn(
                self.q, self.kp, self.vp, self.o1, cfg.B, cfg.H, cfg.N, cfg.Nk, cfg.D, cfg.scale,
                self.dt, s))
        for i in range(len(cfg.schedule)):
            self._timed("dwt_window_plan", lambda: area.area_dwt_window_plan(
                self.src, self.dt, cfg.C, area.AREA_DETAIL_HH, self.energy, self.pcfg[i],
                self.plan[i], self.plan_bytes[i], s))
            self._timed("window_attn", lambda: area.area_window_attn(
                self.q, self.k, self.v, self.pcfg[i], self.plan[i], self.plan_bytes[i],
                self.o2, self.ws, self.ws_bytes, cfg.H, cfg.D, cfg.scale, self.dt, s))

    def window_flops_per_step(self):
        tot, per = 0.0, []
        for p in self.plan:
            d = self.area.parse_plan(p.cpu().numpy())
            f = window_flops(d, self.cfg.H, self.cfg.D)
            per.append(f)
            tot += f
        return tot, per

    def split_fractions(self):
        out = []
        for p in self.plan:
            d = self.area.parse_plan(p.cpu().numpy())
            out.append(round(float(d["split"][0].mean()), 3))
        return out


def call_ms(pairs):
    return [a.elapsed_time(b) for a, b in pairs]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": p.get("hbm_gbs"), "bf16_tflops": p.get("bf16_tflops"),
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def load_traffic(workload: str, kernel_tag: str):
    """DRAM bytes (read + write) per call of a kernel, from the committed ncu
    summary profiles/traffic.json, or None when the summary does not cover this
    workload or was taken from an older build of the kernel."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        t = json.load(fh)
    entry = t.get(workload, {}).get(kernel_tag)
    if not entry or entry.get("kernel_revision") != KERNEL_REVISION:
        return None
    return entry.get("bytes_per_call")


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the same workload
# ---------------------------------------------------------------------------

def oracle_sample(cfg, q, k, v, src, budget_s: float = 15.0, rows_per_call: int = 64):
    """Time the oracle on a sample of the step: all of the DWT map and one
    plan per schedule step, and attention for one head on `rows_per_call`
    query rows per call.  Returns (TFLOP/s of the sampled attention work,
    seconds, description, threads)."""
    from oracle import area_oracle as ora
    t0 = time.perf_counter()
    flops = 0.0
    h = 0
    rng = np.random.default_rng(0)
    E = ora.dwt_detail(src, cfg.Hg, cfg.Wg)
    kp = ora.pool_kv(k[:, h:h + 1], cfg.Hg, cfg.Wg, cfg.f)
    vp = ora.pool_kv(v[:, h:h + 1], cfg.Hg, cfg.Wg, cfg.f)
    rows_per_call = min(rows_per_call, cfg.N)
    rows = np.sort(rng.choice(cfg.N, size=rows_per_call, replace=False))
    ora.coarse_attn(q[:, h:h + 1], kp, vp, cfg.scale, rows=rows)
    flops += 4.0 * rows.size * cfg.Nk * cfg.D
    done_steps = 0
    for w in cfg.schedule:
        if time.perf_counter() - t0 > budget_s:
            break
        plan = ora.window_plan(E[0], cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
        rows = np.sort(rng.choice(cfg.N, size=rows_per_call, replace=False))
        ora.window_attn(q, k, v, [plan], cfg.scale, rows=rows, heads=[h])
        # pairs computed: every window containing a sampled row
        for i, (y0, x0, hy, wx) in enumerate(plan.windows):
            ry, rx = rows // cfg.Wg, rows % cfg.Wg
            inside = np.sum((ry >= y0) & (ry < y0 + hy) & (rx >= x0) & (rx < x0 + wx))
            e = plan.ext[i]
            flops += 4.0 * cfg.D * inside * (e[2] * e[3] + plan.gcount[i])
        done_steps += 1
    sec = time.perf_counter() - t0
    try:
        threads = len(os.sched_getaffinity(0))
    except AttributeError:
        threads = os.cpu_count()
    desc = (f"oracle (NumPy fp64 attention, fp32 exact-order DWT/plan) on {cfg.name}: full "
            f"Haar map, 1 head x {rows_per_call} query rows of one Phase I call, and the plan "
            f"plus 1 head x {rows_per_call} rows of window attention for {done_steps} of "
            f"{len(cfg.schedule)} Phase II steps; TFLOP/s = sampled attention pairs x 4D / time")
    return flops / sec / 1e12, sec, desc, threads


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def l2_note(cfg) -> str:
    tensor = cfg.B * cfg.H * cfg.N * cfg.D * (2 if cfg.dtype == "bf16" else 4)
    rel = "larger" if tensor > 126e6 else "smaller"
    return f"inputs {rel} than L2 ({tensor / 1e9:.2f} GB per Q/K/V tensor, L2 126 MB)"


def workload_config(cfg, heads: int, world: int, sharded: bool) -> dict:
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": cfg.name, "grid": [cfg.Hg, cfg.Wg], "tokens": cfg.N,
            "heads": heads, "head_dim": cfg.D, "batch": cfg.B, "pool_f": cfg.f,
            "schedule": list(cfg.schedule), "halo": cfg.halo, "G": cfg.G,
            "split_thr": cfg.split_thr, "phase1_calls": len(cfg.schedule),
            "phase2_calls": len(cfg.schedule),
            "l2": l2_note(cfg),
            "parallelism": (f"heads sharded over {world} GPUs, {-(-heads // world)} or fewer "
                            "per GPU" if sharded else f"replicas x{world}")}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from workloads import CONFIGS, make_detail_source, make_qkv
    cfg = CONFIGS[args.config]
    q, k, v = make_qkv(cfg)
    src = make_detail_source(cfg)
    for _ in range(args.warmup):
        oracle_sample(cfg, q, k, v, src, budget_s=args.ref_budget / 4, rows_per_call=16)
    vals, secs = [], []
    desc, threads = "", 0
    for _ in range(args.steps):
        val, sec, desc, threads = oracle_sample(cfg, q, k, v, src, budget_s=args.ref_budget,
                                                rows_per_call=32)
        vals.append(val)
        secs.append(sec)
    value = float(np.median(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * float(np.median(secs)), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg, cfg.H, args.gpus, False),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def schedule_graph_leg(cfg, st, stream, full_ms, steps=28, shift=3.0, sigma_star=0.89):
    """A whole sampling run of attention calls: the noise-level phase switch
    over a synthetic flow-matching sampler, the pooling ramp over the Phase I
    steps and the shrinking windows over the Phase II steps, captured once in
    one CUDA graph and replayed.  Returns the summary for the JSON line."""
    import torch

    import step_adaptive_sparse_b200 as area
    from workloads import flow_sigmas
    dev = st.q.device
    sig = flow_sigmas(steps, shift)
    sched = area.area_schedule(sig, sigma_star, cfg.f, 2, cfg.schedule[0], cfg.schedule[-1],
                               cfg.Hg, cfg.Wg)
    fs = [p for kd, p in sched if kd == area.AREA_PHASE_COARSE]
    ws_sides = [p for kd, p in sched if kd == area.AREA_PHASE_WINDOW]
    nk_max = max([(cfg.Hg // f) * (cfg.Wg // f) for f in fs], default=1)
    kp = torch.empty((cfg.B, cfg.H, nk_max, cfg.D), dtype=st.q.dtype, device=dev)
    vp = torch.empty_like(kp)
    plans = {}
    wsb = 0
    for w in sorted(set(ws_sides)):
        pc = area.make_cfg(cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
        nb = area.area_window_plan_bytes(pc)
        wsb = max(wsb, area.area_window_attn_ws_bytes(pc, cfg.H, cfg.D)
                  + area.area_window_attn_stage_bytes(pc, cfg.H, cfg.D))
        plans[w] = (pc, torch.empty(nb, dtype=torch.uint8, device=dev), nb)
    # the run's window sides overlap differently from the step's: own workspace
    ws = torch.empty(wsb // 4, dtype=torch.float32, device=dev)

    def run():
        for kd, p in sched:
            if kd == area.AREA_PHASE_COARSE:
                nk = (cfg.Hg // p) * (cfg.Wg // p)
                area.area_pool_kv(st.k, st.v, kp, vp, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, p,
                                  area.AREA_POOL_MEAN, st.dt, stream)
                area.area_coarse_attn(st.q, kp, vp, st.o1, cfg.B, cfg.H, cfg.N, nk, cfg.D,
                                      cfg.scale, st.dt, stream)
            else:
                pc, plan, nb = plans[p]
                area.area_dwt_window_plan(st.src, st.dt, cfg.C, area.AREA_DETAIL_HH, st.energy,
                                          pc, plan, nb, stream)
                area.area_window_attn(st.q, st.k, st.v, pc, plan, nb, st.o2, ws, wsb,
                                      cfg.H, cfg.D, cfg.scale, st.dt, stream)

    with torch.cuda.stream(stream):
        run()                                       # eager pass: capture warm-up, plans
    torch.cuda.synchronize()
    flops = sum(4.0 * cfg.B * cfg.H * cfg.N * (cfg.Hg // f) * (cfg.Wg // f) * cfg.D for f in fs)
    wfl = {w: window_flops(area.parse_plan(pl.cpu().numpy()), cfg.H, cfg.D)
           for w, (_, pl, _) in plans.items()}
    flops += sum(wfl[w] for w in ws_sides)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    g.replay()
    torch.cuda.synchronize()
    reps = 2
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):                 # replay() launches on the current stream
        for _ in range(reps):
            g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del g
    launches = 2 * len(fs) + len(ws_sides) * (1 + WINDOW_LAUNCHES)
    return {"steps": steps, "sampler": f"flow matching, shift {shift}", "sigma_star": sigma_star,
            "phase1_steps": len(fs), "ramp": fs, "window_sides": ws_sides,
            "graph_launches": launches, "ms": ms,
            "tflops": flops / (ms * 1e-3) / 1e12,
            "speedup_vs_full_attention": steps * full_ms / ms,
            "note": "all attention calls of the run captured in one CUDA graph; "
                    "speedup against the same number of full-attention calls"}


def config_leg(name: str, dev, stream, steps: int = 3, warmup: int = 3) -> dict:
    """The metric's other configuration, timed like the main step (the same
    call sequence, CUDA events on the launching stream, inputs larger than L2)
    and reported per call: Phase I and Phase II ms and TFLOP/s, and the window
    calls' fraction of the measured sustained bf16 peak."""
    import torch

    from workloads import CONFIGS, make_detail_source, make_qkv
    cfg = CONFIGS[name]
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    q, k, v = (torch.from_numpy(x).to(dev).to(tdt) for x in make_qkv(cfg))
    src = torch.from_numpy(make_detail_source(cfg)).to(dev).to(tdt)
    st = AreaStep(cfg, q, k, v, src, stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            st.run()
    torch.cuda.synchronize()
    wfl, wper = st.window_flops_per_step()
    st.record = True
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            st.run()
    e1.record(stream)
    torch.cuda.synchronize()
    st.record = False
    ms = e0.elapsed_time(e1) / steps
    per = {n: call_ms(p) for n, p in st.calls.items()}
    coarse_ms = float(np.median(per["coarse_attn"]))
    win_ms = np.array(per["window_attn"]).reshape(steps, -1).mean(axis=0)
    step_flops = phase1_flops(cfg) * st.n_phase1 + wfl
    peak = load_peaks()["bf16_tflops_sustained"]
    win_tf = wfl / (float(win_ms.sum()) * 1e-3) / 1e12
    out = {"workload": name, "steps": steps, "warmup": warmup, "ms_per_step": ms,
           "value": step_flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
           "coarse_attn_ms": coarse_ms,
           "coarse_attn_tflops": phase1_flops(cfg) / (coarse_ms * 1e-3) / 1e12,
           "window_attn_ms_by_step": win_ms.tolist(),
           "window_attn_tflops_by_step": [f / (t * 1e-3) / 1e12 for f, t in zip(wper, win_ms)],
           "window_attn_tflops": win_tf,
           "window_frac_of_sustained_peak": win_tf / peak,
           "coarse_frac_of_sustained_peak": phase1_flops(cfg) / (coarse_ms * 1e-3) / 1e12 / peak,
           "dwt_window_plan_ms": float(np.median(per["dwt_window_plan"])),
           "pool_kv_gbs": pool_bytes(cfg) / (float(np.median(per["pool_kv"])) * 1e-3) / 1e9,
           "split_fraction_by_step": st.split_fractions()}
    del st, q, k, v, src
    torch.cuda.empty_cache()
    return out


def profile_pass(args) -> int:
    """Every kernel of the path, twice, on one configuration: the input of the
    per-kernel ncu captures (a capture selects the second launch of a kernel
    with -s/-c).  Sequence per pass: pool_kv, coarse attention, the detail
    map, the separate planner, the one-launch planner (once per window step),
    window attention at schedule step --profile-step (or one call per step of
    --profile-steps), bridge selection and bridged window attention.  Nothing
    is timed."""
    import torch

    import step_adaptive_sparse_b200 as area
    from workloads import CONFIGS, make_detail_source, make_qkv
    cfg = CONFIGS[args.config]
    dev = torch.device("cuda", 0)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    q, k, v = (torch.from_numpy(x).to(dev).to(tdt) for x in make_qkv(cfg))
    src = torch.from_numpy(make_detail_source(cfg)).to(dev).to(tdt)
    stream = torch.cuda.Stream(device=dev)
    st = AreaStep(cfg, q, k, v, src, stream)
    steps = ([int(x) % len(cfg.schedule) for x in args.profile_steps.split(",")]
             if args.profile_steps else [args.profile_step % len(cfg.schedule)])
    i = steps[-1]
    w = cfg.schedule[i]
    ry, rx = area.area_bridge_lattice(w, cfg.Hg, cfg.Wg)
    cand = torch.empty((cfg.B, cfg.H, ry * rx), dtype=torch.int32, device=dev)
    mws = torch.empty(area.area_bridge_select_ws_bytes(cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D) // 4,
                      dtype=torch.float32, device=dev)
    s = stream
    with torch.cuda.stream(stream):
        for _ in range(2):
            area.area_pool_kv(k, v, st.kp, st.vp, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, cfg.f,
                              area.AREA_POOL_MEAN, st.dt, s)
            area.area_coarse_attn(q, st.kp, st.vp, st.o1, cfg.B, cfg.H, cfg.N, cfg.Nk, cfg.D,
                                  cfg.scale, st.dt, s)
            area.area_dwt_detail(src, st.dt, cfg.C, st.energy, cfg.B, cfg.Hg, cfg.Wg,
                                 area.AREA_DETAIL_HH, s)
            area.area_window_plan(st.energy, st.pcfg[i], st.plan[i], st.plan_bytes[i], s)
            for si in steps:
                area.area_dwt_window_plan(src, st.dt, cfg.C, area.AREA_DETAIL_HH, st.energy,
                                          st.pcfg[si], st.plan[si], st.plan_bytes[si], s)
            for si in steps:
                area.area_window_attn(q, k, v, st.pcfg[si], st.plan[si], st.plan_bytes[si], st.o2,
                                      st.ws, st.ws_bytes, cfg.H, cfg.D, cfg.scale, st.dt, s)
            area.area_bridge_select(k, st.dt, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, ry, rx, cand,
                                    mws, mws.numel() * 4, s)
            area.area_window_attn_bridge(q, k, v, cand, ry * rx, st.pcfg[i], st.plan[i],
                                         st.plan_bytes[i], st.o2, st.ws, st.ws_bytes, cfg.H,
                                         cfg.D, cfg.scale, st.dt, s)
    torch.cuda.synchronize()
    err = area.area_kernel_error()
    print(json.dumps({"profile_pass": cfg.name, "window_sides": [cfg.schedule[si] for si in steps],
                      "kernel_error": err}))
    return 0 if err == 0 else 1


def run_area(args):
    import torch

    import step_adaptive_sparse_b200 as area
    from workloads import CONFIGS, make_detail_source, make_qkv
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (libarea has no CPU path)")
    torch.cuda.set_device(local)
    dist = init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    cfg = CONFIGS[args.config]
    qh, kh, vh = make_qkv(cfg)
    srch = make_detail_source(cfg)
    sharded = args.shard == "heads" and world > 1
    H_all = cfg.H
    if sharded:
        # strong scaling: this rank computes its heads of the one problem
        from dataclasses import replace
        h0, h1 = head_range(rank, world, cfg.H)
        qh, kh, vh = (np.ascontiguousarray(x[:, h0:h1]) for x in (qh, kh, vh))
        cfg = replace(cfg, H=h1 - h0)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    # pinned host copies for the end-to-end leg
    pin = [torch.from_numpy(x).to(tdt).pin_memory() for x in (qh, kh, vh, srch)]
    q, k, v, src = (p.to(dev, non_blocking=False) for p in pin)
    stream = torch.cuda.Stream(device=dev)
    st = AreaStep(cfg, q, k, v, src, stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            st.run()
    torch.cuda.synchronize()
    # every rank learns of a bounded-wait expiry on any rank, and all stop
    # together instead of leaving the others in the next collective
    kerr = reduce_max(dist, float(area.area_kernel_error()), device=str(dev))
    if kerr:
        if dist is not None:
            dist.destroy_process_group()
        raise SystemExit("bench.py: a kernel gave up a bounded wait in warm-up")
    win_flops, win_per_step = st.window_flops_per_step()
    splits = st.split_fractions()
    step_flops = phase1_flops(cfg) * st.n_phase1 + win_flops

    # ---- timed region (device time, CUDA events on the launching stream)
    st.record = True
    barrier(dist, local)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, args.clocks_csv) as clocks:
        time.sleep(0.3)
        ev0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                st.run()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(dist, local)
    st.record = False
    ms_local = ev0.elapsed_time(ev1)
    ms_total = reduce_max(dist, ms_local, device=str(dev))
    ms_step = ms_total / args.steps
    flops_all = reduce_sum(dist, step_flops * args.steps, device=str(dev))
    value = flops_all / (ms_total * 1e-3) / 1e12

    per = {n: call_ms(p) for n, p in st.calls.items()}
    med = {n: (float(np.median(x)) if x else None) for n, x in per.items()}
    win_ms_steps = np.array(per["window_attn"]).reshape(args.steps, -1).mean(axis=0).tolist()
    kerr = area.area_kernel_error()

    # ---- the same step captured once in a CUDA graph and replayed
    graph_ms = None
    if not args.no_graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            st.run()
        g.replay()
        torch.cuda.synchronize()
        ge0, ge1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ge0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                g.replay()
        ge1.record(stream)
        torch.cuda.synchronize()
        graph_ms = ge0.elapsed_time(ge1) / args.steps
        del g

    # ---- full attention: the speedup denominator (same inputs)
    o_full = torch.empty_like(q)
    fe0, fe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        area.area_full_attn(q, k, v, o_full, cfg.B, cfg.H, cfg.N, cfg.D, cfg.scale, st.dt, stream)
        fe0.record(stream)
        for _ in range(args.full_reps):
            area.area_full_attn(q, k, v, o_full, cfg.B, cfg.H, cfg.N, cfg.D, cfg.scale, st.dt,
                                stream)
        fe1.record(stream)
    torch.cuda.synchronize()
    full_ms = fe0.elapsed_time(fe1) / args.full_reps
    del o_full

    # ---- Phase I with the pages' pooling ramp (f0 -> 2 over the 8 steps),
    # measured once after the timed region (the configs' step uses a fixed f)
    ramp = area.area_pool_ramp(cfg.f, 2, st.n_phase1, cfg.Hg, cfg.Wg)
    nk_max = (cfg.Hg // min(ramp)) * (cfg.Wg // min(ramp))
    kp_r = torch.empty((cfg.B, cfg.H, nk_max, cfg.D), dtype=q.dtype, device=dev)
    vp_r = torch.empty_like(kp_r)
    o_r = torch.empty_like(q)
    ramp_ms, ramp_tf = [], []
    with torch.cuda.stream(stream):
        for rep in range(2):                       # warm-up pass, then the timed pass
            for f in ramp:
                nk = (cfg.Hg // f) * (cfg.Wg // f)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                area.area_pool_kv(k, v, kp_r, vp_r, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, f,
                                  area.AREA_POOL_MEAN, st.dt, stream)
                area.area_coarse_attn(q, kp_r, vp_r, o_r, cfg.B, cfg.H, cfg.N, nk, cfg.D,
                                      cfg.scale, st.dt, stream)
                b.record(stream)
                if rep:
                    ramp_ms.append((a, b, 4.0 * cfg.B * cfg.H * cfg.N * nk * cfg.D))
    torch.cuda.synchronize()
    ramp_out = {"ramp": ramp, "ms": [], "tflops": []}
    for a, b, fl in ramp_ms:
        t = a.elapsed_time(b)
        ramp_out["ms"].append(t)
        ramp_out["tflops"].append(fl / (t * 1e-3) / 1e12)
    ramp_out["total_ms"] = float(sum(ramp_out["ms"]))
    del kp_r, vp_r, o_r

    # ---- the pages' own bridge rule on the last (smallest) window size:
    # candidate selection plus window attention, median of 4 timed repetitions
    # after one untimed
    w_b = cfg.schedule[-1]
    ry, rx = area.area_bridge_lattice(w_b, cfg.Hg, cfg.Wg)
    cand = torch.empty((cfg.B, cfg.H, ry * rx), dtype=torch.int32, device=dev)
    mws = torch.empty(area.area_bridge_select_ws_bytes(cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D) // 4,
                      dtype=torch.float32, device=dev)
    pc0 = area.make_cfg(cfg.B, cfg.Hg, cfg.Wg, w_b, cfg.halo, 0, cfg.split_thr)
    nb0 = area.area_window_plan_bytes(pc0)
    plan0 = torch.empty(nb0, dtype=torch.uint8, device=dev)
    bridge_out = {}
    with torch.cuda.stream(stream):
        area.area_dwt_detail(src, st.dt, cfg.C, st.energy, cfg.B, cfg.Hg, cfg.Wg,
                             area.AREA_DETAIL_HH, stream)
        area.area_window_plan(st.energy, pc0, plan0, nb0, stream)
        bev = []
        for rep in range(5):
            a, b2, c2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a.record(stream)
            area.area_bridge_select(k, st.dt, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, ry, rx, cand,
                                    mws, mws.numel() * 4, stream)
            b2.record(stream)
            area.area_window_attn_bridge(q, k, v, cand, ry * rx, pc0, plan0, nb0, st.o2, st.ws,
                                         st.ws_bytes, cfg.H, cfg.D, cfg.scale, st.dt, stream)
            c2.record(stream)
            if rep > 0:
                bev.append((a, b2, c2))
    torch.cuda.synchronize()
    d0 = area.parse_plan(plan0.cpu().numpy())
    cnd = cand.cpu().numpy().astype(np.int64)
    pairs = 0.0
    nwin0 = int(d0["nwin"][0])
    for i in range(nwin0):
        y0, x0, hy, wx = (int(t) for t in d0["win"][0, i])
        ey0, ex0, ehy, ewx = (int(t) for t in d0["ext"][0, i])
        cy, cx = cnd[0] // cfg.Wg, cnd[0] % cfg.Wg                # [H, R]
        outside = ~((cy >= ey0) & (cy < ey0 + ehy) & (cx >= ex0) & (cx < ex0 + ewx))
        pairs += hy * wx * (ehy * ewx * cfg.H + float(outside.sum()))
    bflops = 4.0 * cfg.D * cfg.B * pairs
    battn_ms = float(np.median([b_.elapsed_time(c_) for a_, b_, c_ in bev]))
    sel_ms = float(np.median([a_.elapsed_time(b_) for a_, b_, c_ in bev]))
    k_bytes = float(k.numel() * k.element_size())
    bridge_out = {"window": w_b, "lattice": [ry, rx], "select_ms": sel_ms,
                  "select_gbs": 2.0 * k_bytes / (sel_ms * 1e-3) / 1e9,
                  "select_note": "algorithmic bytes: K read twice (chunk sums, then deviations)",
                  "window_attn_ms": battn_ms,
                  "window_attn_tflops": bflops / (battn_ms * 1e-3) / 1e12}
    del cand, mws, plan0

    # ---- detail map + planner: one cooperative launch against the separate
    # calls, at the last schedule step (eager, 10 calls each)
    fused = {}
    with torch.cuda.stream(stream):
        i_last = len(cfg.schedule) - 1
        pc_l, pl_l, nb_l = st.pcfg[i_last], st.plan[i_last], st.plan_bytes[i_last]
        for tag in ("separate", "fused"):
            def call():
                if tag == "fused":
                    area.area_dwt_window_plan(st.src, st.dt, cfg.C, area.AREA_DETAIL_HH, st.energy,
                                              pc_l, pl_l, nb_l, stream)
                else:
                    area.area_dwt_detail(st.src, st.dt, cfg.C, st.energy, cfg.B, cfg.Hg, cfg.Wg,
                                         area.AREA_DETAIL_HH, stream)
                    area.area_window_plan(st.energy, pc_l, pl_l, nb_l, stream)
            for _ in range(3):
                call()
            fa, fb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            fa.record(stream)
            for _ in range(10):
                call()
            fb.record(stream)
            torch.cuda.synchronize()
            fused[tag + "_us"] = fa.elapsed_time(fb) / 10 * 1e3
    fused["launches"] = {"separate": 1 + plan_launches(cfg.B), "fused": 1}

    # ---- the detail map alone, for its HBM figure: L2 is flushed (a 256 MB
    # write, twice the L2) before each call so the source comes from HBM
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    dwt_pairs = []
    with torch.cuda.stream(stream):
        for rep in range(13):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            area.area_dwt_detail(st.src, st.dt, cfg.C, st.energy, cfg.B, cfg.Hg, cfg.Wg,
                                 area.AREA_DETAIL_HH, stream)
            b.record(stream)
            if rep >= 3:
                dwt_pairs.append((a, b))
    torch.cuda.synchronize()
    dwt_ms = float(np.median(call_ms(dwt_pairs)))
    del flush

    # ---- a whole 28-step sampling run in one CUDA graph
    sched_out = None if args.no_graph else schedule_graph_leg(cfg, st, stream, full_ms)

    # ---- end to end through the C-ABI from pinned host buffers.  Each step
    # copies its inputs host->device and its output device->host; two device
    # buffer sets let the copies of one step overlap the kernels of the next
    # (one stream per copy direction), as a serving loop would.
    out_h = torch.empty(q.shape, dtype=tdt).pin_memory()
    h2d = sum(p.numel() * p.element_size() for p in pin)
    d2h = out_h.numel() * out_h.element_size()
    sets = [(q, k, v, src, st.o2),
            tuple(torch.empty_like(t) for t in (q, k, v, src, st.o2))]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)
    ev_in, ev_used, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def upload(i):
        s_in.wait_event(ev_used[i])          # the kernels of step i-2 are done with set i
        with torch.cuda.stream(s_in):
            for dst_t, src_t in zip(sets[i][:4], pin):
                dst_t.copy_(src_t, non_blocking=True)
        ev_in[i].record(s_in)

    barrier(dist, local)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    upload(0)
    for step in range(args.steps):
        cur = step % 2
        if step + 1 < args.steps:
            upload(1 - cur)
        stream.wait_event(ev_in[cur])
        stream.wait_event(ev_out[cur])           # step-2's output has left this buffer
        st.q, st.k, st.v, st.src, st.o2 = sets[cur]
        with torch.cuda.stream(stream):
            st.run()
        ev_used[cur].record(stream)
        s_out.wait_event(ev_used[cur])
        with torch.cuda.stream(s_out):
            out_h.copy_(sets[cur][4], non_blocking=True)
        ev_out[cur].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize()
    st.q, st.k, st.v, st.src, st.o2 = sets[0]
    del sets
    e2e_ms = reduce_max(dist, e0.elapsed_time(e1), device=str(dev))
    e2e_val = flops_all / (e2e_ms * 1e-3) / 1e12

    # ---- the metric's other configuration (4096^2), reported per call
    other = None
    if world == 1 and args.config == DEFAULT_CONFIG and args.other_config:
        other = config_leg(args.other_config, dev, stream)

    # ---- roofline of the dominant kernel
    peaks = load_peaks()
    n1 = st.n_phase1
    coarse_ms = med["coarse_attn"]
    t_coarse = coarse_ms * n1
    t_window = float(np.sum(win_ms_steps))
    if t_window >= t_coarse:
        dom, dom_flops, dom_ms, dom_launches = ("window_attn", win_flops / len(cfg.schedule),
                                                t_window / len(cfg.schedule),
                                                "the global-KV staging copy and the attention kernel, after a 256-byte memset; timed together")
    else:
        dom, dom_flops, dom_ms, dom_launches = ("coarse_attn", phase1_flops(cfg), coarse_ms,
                                                "1 launch")
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak,
            "traffic": None if sharded else load_traffic(cfg.name, dom),
            "kernel": dom, "per_call": dom_launches,
            "peak_kind": f"bf16 dense, {peaks['source']} sustained",
            "frac_of_burst_peak": achieved / peaks["bf16_tflops"],
            # the B200's published dense bf16 rate (2.25 PFLOP/s), for reference
            "frac_of_published_peak": achieved / PUBLISHED_BF16_TFLOPS}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # about 10 s of the host's cores: 8192 query rows per sampled call
        val, sec, desc, threads = oracle_sample(cfg, qh, kh, vh, srch, budget_s=args.ref_budget,
                                                rows_per_call=8192)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": desc, "seconds": sec}

    clk = clocks.summary()
    if rank == 0:
        pool_ms = med["pool_kv"]
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None,
            "dtype": "bf16" if cfg.dtype == "bf16" else "f32", "data": "synthetic",
            "config": workload_config(cfg, H_all, world, sharded),
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps},
            "gpu_launches": st.launches * args.steps,
            "clocks": clk,
            "kernel_error": kerr,
            "per_call_ms": {
                "pool_kv": pool_ms, "coarse_attn": coarse_ms, "dwt_detail_alone": dwt_ms,
                "dwt_window_plan": med["dwt_window_plan"], "window_attn_by_step": win_ms_steps,
                "full_attn": full_ms},
            "per_call_tflops": {
                "coarse_attn": phase1_flops(cfg) / (coarse_ms * 1e-3) / 1e12,
                "window_attn_by_step": [f / (t * 1e-3) / 1e12 for f, t in
                                        zip(win_per_step, win_ms_steps)],
                "full_attn": full_flops(cfg) / (full_ms * 1e-3) / 1e12},
            "per_call_gbs": {"pool_kv": pool_bytes(cfg) / (pool_ms * 1e-3) / 1e9,
                             "dwt_detail_alone": dwt_bytes(cfg) / (dwt_ms * 1e-3) / 1e9,
                             "hbm_peak_gbs": peaks["hbm_gbs"]},
            "split_fraction_by_step": splits,
            "phase1_pooling_ramp": ramp_out,
            "pages_bridge_rule": bridge_out,
            "schedule_28_steps_graph": sched_out,
            "dwt_plan_one_launch": fused,
            "other_config": other,
            "graph_replay": None if graph_ms is None else {
                "ms_per_step": graph_ms,
                "value": step_flops / (graph_ms * 1e-3) / 1e12,
                "note": f"the same step captured once in a CUDA graph ({st.launches} launches) "
                        "and replayed"},
            "speedup_vs_full_attention": (full_ms * (n1 + len(cfg.schedule))) / ms_step,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["area", "reference"], default="area")
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--full-reps", type=int, default=2)
    ap.add_argument("--ref-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--other-config", default="flux4096",
                    help="the metric's second configuration, timed after the main one at "
                         "N = 1 (empty string: skip)")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay leg")
    ap.add_argument("--clocks-csv", default="",
                    help="where to keep the nvidia-smi clock samples of the timed region "
                         "(default: the system temporary directory)")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: independent replicas (weak scaling) or the heads of one "
                         "problem split across ranks (strong scaling)")
    ap.add_argument("--profile-pass", action="store_true",
                    help="run every kernel of the path twice on --config, untimed (the "
                         "input of the per-kernel ncu captures)")
    ap.add_argument("--profile-step", type=int, default=-1,
                    help="schedule step of the window calls in --profile-pass")
    ap.add_argument("--profile-steps", default="",
                    help="comma-separated schedule steps: one window call each per pass "
                         "(overrides --profile-step)")
    args = ap.parse_args(argv)
    if args.profile_pass:
        return profile_pass(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_area(args)


if __name__ == "__main__":
    sys.exit(main())
