"""A whole AReA schedule step captured in one CUDA graph and replayed.

Every libarea call is asynchronous on the caller's stream and never reads the
device from the host (the plan stays on the device), so a step of both phases
can be captured once and replayed: the replay must reproduce the eager
results (window outputs up to the order of fp32 additions in overlaps).
"""
import numpy as np
import pytest
import torch

import step_adaptive_sparse_b200 as area
from workloads import CONFIGS, make_detail_source, make_qkv

pytestmark = pytest.mark.gpu


def _step(bufs, cfg, dt, stream):
    q, k, v, src, kp, vp, o1, o2, energy, plans, ws, wsb = bufs
    area.area_pool_kv(k, v, kp, vp, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, cfg.f,
                      area.AREA_POOL_MEAN, dt, stream)
    area.area_coarse_attn(q, kp, vp, o1, cfg.B, cfg.H, cfg.N, cfg.Nk, cfg.D, cfg.scale, dt, stream)
    for (pc, plan, nb), o in zip(plans, o2):
        area.area_dwt_detail(src, dt, cfg.C, energy, cfg.B, cfg.Hg, cfg.Wg, area.AREA_DETAIL_HH,
                             stream)
        area.area_window_plan(energy, pc, plan, nb, stream)
        area.area_window_attn(q, k, v, pc, plan, nb, o, ws, wsb, cfg.H, cfg.D, cfg.scale, dt,
                              stream)


@pytest.mark.parametrize("name", ["tiny", "flux2048"])
def test_schedule_step_graph_replay_matches_eager(name):
    cfg = CONFIGS[name]
    dt = area.AREA_DTYPE_BF16 if cfg.dtype == "bf16" else area.AREA_DTYPE_F32
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    q, k, v = (torch.from_numpy(x).cuda().to(tdt) for x in make_qkv(cfg))
    src = torch.from_numpy(make_detail_source(cfg)).cuda().to(tdt)
    kp = torch.empty((cfg.B, cfg.H, cfg.Nk, cfg.D), dtype=tdt, device="cuda")
    vp = torch.empty_like(kp)
    energy = torch.empty((cfg.B, cfg.Hg // 2, cfg.Wg // 2), dtype=torch.float32, device="cuda")
    plans, wsb = [], 0
    for w in cfg.schedule:
        pc = area.make_cfg(cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
        nb = area.area_window_plan_bytes(pc)
        plans.append((pc, torch.empty(nb, dtype=torch.uint8, device="cuda"), nb))
        wsb = max(wsb, area.area_window_attn_ws_bytes(pc, cfg.H, cfg.D)
                  + area.area_window_attn_stage_bytes(pc, cfg.H, cfg.D))
    ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
    o1 = torch.empty_like(q)
    o2 = [torch.empty_like(q) for _ in cfg.schedule]
    bufs = (q, k, v, src, kp, vp, o1, o2, energy, plans, ws, wsb)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        _step(bufs, cfg, dt, stream)            # eager, also the capture warm-up
    torch.cuda.synchronize()
    ref1 = o1.clone()
    ref2 = [o.clone() for o in o2]
    ref_plans = [p.clone() for _, p, _ in plans]
    for t in [o1] + o2 + [p for _, p, _ in plans]:
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        _step(bufs, cfg, dt, stream)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o1, ref1)
    for (_, p, _), rp in zip(plans, ref_plans):
        assert torch.equal(p[:256], rp[:256])
    # the merge of overlapped tokens runs in a fixed order: replays are
    # bit-identical to the eager run
    for o, r in zip(o2, ref2):
        assert torch.equal(o, r)
    assert area.area_kernel_error() == 0
    del g


@pytest.mark.parametrize("name", ["tiny", "flux2048", "flux6144"])
def test_one_launch_planner_in_a_graph(name):
    # the cooperative detail map + planner launch (and the reset of its
    # barrier words) captured in a graph: replay == eager, byte for byte
    cfg = CONFIGS[name]
    dt = area.AREA_DTYPE_BF16 if cfg.dtype == "bf16" else area.AREA_DTYPE_F32
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    src = torch.from_numpy(make_detail_source(cfg)).cuda().to(tdt)
    energy = torch.empty((cfg.B, cfg.Hg // 2, cfg.Wg // 2), dtype=torch.float32, device="cuda")
    plans = []
    for w in cfg.schedule:
        pc = area.make_cfg(cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
        nb = area.area_window_plan_bytes(pc)
        # zero-filled: the 256-byte padding after each section is never written
        plans.append((pc, torch.zeros(nb, dtype=torch.uint8, device="cuda"), nb))
    stream = torch.cuda.Stream()

    def run():
        for pc, plan, nb in plans:
            area.area_dwt_window_plan(src, dt, cfg.C, area.AREA_DETAIL_HH, energy, pc, plan, nb,
                                      stream)

    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    ends = []
    for _, p, _ in plans:
        hdr = p[:256].cpu().numpy().view(np.int64)
        ends.append(int(hdr[10 + area.SECTIONS.index("SCRATCH")]))
    ref = [p[:e].clone() for (_, p, _), e in zip(plans, ends)]
    ref_e = energy.clone()
    for _, p, _ in plans:
        p.zero_()
    energy.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert area.area_kernel_error() == 0
    assert torch.equal(energy.view(torch.int32), ref_e.view(torch.int32))
    for (_, p, _), e, r in zip(plans, ends, ref):
        assert torch.equal(p[:e], r)
    del g


def test_whole_sampling_run_in_one_graph():
    # 28 steps of a synthetic flow-matching sampler: the noise-level switch,
    # the pooling ramp over Phase I and the shrinking windows over Phase II,
    # every call of the run captured in one graph
    from workloads import flow_sigmas
    cfg = CONFIGS["flux2048"]
    dt = area.AREA_DTYPE_BF16
    q, k, v = (torch.from_numpy(x).cuda().to(torch.bfloat16) for x in make_qkv(cfg))
    src = torch.from_numpy(make_detail_source(cfg)).cuda().to(torch.bfloat16)
    sched = area.area_schedule(flow_sigmas(28, 3.0), 0.89, 4, 2, 64, 32, cfg.Hg, cfg.Wg)
    kinds = [kd for kd, _ in sched]
    assert kinds == [area.AREA_PHASE_COARSE] * 8 + [area.AREA_PHASE_WINDOW] * 20
    fs = [p for kd, p in sched if kd == area.AREA_PHASE_COARSE]
    assert fs == [4, 4, 4, 4, 2, 2, 2, 2]
    kp = torch.empty((cfg.B, cfg.H, cfg.N // 4, cfg.D), dtype=torch.bfloat16, device="cuda")
    vp = torch.empty_like(kp)
    energy = torch.empty((cfg.B, cfg.Hg // 2, cfg.Wg // 2), dtype=torch.float32, device="cuda")
    plans, wsb = {}, 0
    for w in {p for kd, p in sched if kd == area.AREA_PHASE_WINDOW}:
        pc = area.make_cfg(cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
        nb = area.area_window_plan_bytes(pc)
        plans[w] = (pc, torch.empty(nb, dtype=torch.uint8, device="cuda"), nb)
        wsb = max(wsb, area.area_window_attn_ws_bytes(pc, cfg.H, cfg.D)
                  + area.area_window_attn_stage_bytes(pc, cfg.H, cfg.D))
    ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    outs1, outs2 = [], []

    def run(keep):
        for kd, p in sched:
            if kd == area.AREA_PHASE_COARSE:
                nk = (cfg.Hg // p) * (cfg.Wg // p)
                area.area_pool_kv(k, v, kp, vp, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, p,
                                  area.AREA_POOL_MEAN, dt, stream)
                area.area_coarse_attn(q, kp, vp, o1, cfg.B, cfg.H, cfg.N, nk, cfg.D, cfg.scale,
                                      dt, stream)
                if keep:
                    outs1.append(o1.clone())
            else:
                pc, plan, nb = plans[p]
                area.area_dwt_detail(src, dt, cfg.C, energy, cfg.B, cfg.Hg, cfg.Wg,
                                     area.AREA_DETAIL_HH, stream)
                area.area_window_plan(energy, pc, plan, nb, stream)
                area.area_window_attn(q, k, v, pc, plan, nb, o2, ws, wsb, cfg.H, cfg.D,
                                      cfg.scale, dt, stream)
                if keep:
                    outs2.append(o2.clone())

    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        run(True)                                   # eager, per-step outputs kept
    torch.cuda.synchronize()
    o1.zero_()
    o2.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run(False)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o1, outs1[-1])               # last Phase I step (f = 2)
    assert torch.equal(o2, outs2[-1])               # fixed-order merge: bit-identical
    assert not torch.equal(outs1[0], outs1[-1])     # the ramp changed the pooled grid
    assert area.area_kernel_error() == 0
    del g
