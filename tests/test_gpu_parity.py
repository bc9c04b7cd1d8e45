"""GPU parity: the CUDA path through the C-ABI against the CPU oracle.

Bars: index plans, split decisions, scores, global-KV lists, merge-weight sums
and detail maps bit-exact; attention outputs within max-abs 2e-2 / mean-abs
2e-3 for bf16 inputs (fp32 accumulation) and 1e-4 for fp32.  Full-size
configurations are checked on sampled query rows: a row's output depends only
on its own query, so the per-row comparison is exact in what it checks.
"""
import numpy as np
import pytest
import torch

from oracle import area_oracle as ora
from workloads import CONFIGS, make_text_kv
import gpu_runner as gr

pytestmark = pytest.mark.gpu

BIG = ["flux2048", "flux4096", "flux6144", "qwen6144x2048"]
ALL = ["tiny"] + BIG


def _steps(name):
    return list(range(len(CONFIGS[name].schedule)))


# ---------------------------------------------------------------------------
# DWT detail map: bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ALL)
def test_dwt_bitexact(name):
    cfg = CONFIGS[name]
    src = gr.host_src(name)
    dsrc = gr.to_dev(src, cfg.dtype)
    for mode, mname in [(0, "hh"), (1, "all3")]:
        got = gr.gpu_dwt(dsrc, cfg.B, cfg.Hg, cfg.Wg, cfg.C, cfg.dtype, mode).cpu().numpy()
        want = ora.dwt_detail(src, cfg.Hg, cfg.Wg, mname)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (name, mname)


@pytest.mark.parametrize("C,Hg,Wg,dtype", [(3, 10, 6, "fp32"), (5, 8, 14, "bf16"),
                                           (16, 2, 2, "bf16"), (8, 34, 18, "fp32")])
def test_dwt_odd_channels_and_small_grids(C, Hg, Wg, dtype):
    rng = np.random.default_rng(C * 100 + Hg)
    src = rng.standard_normal((2, Hg * Wg, C)).astype(np.float32)
    if dtype == "bf16":
        src = gr.to_host(gr.to_dev(src, "bf16")).astype(np.float32)
    got = gr.gpu_dwt(gr.to_dev(src, dtype), 2, Hg, Wg, C, dtype).cpu().numpy()
    want = ora.dwt_detail(src, Hg, Wg, "hh")
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


# ---------------------------------------------------------------------------
# Planner: bit-exact at every configuration and schedule step
# ---------------------------------------------------------------------------

def _check_items(got, want, b=0):
    nitem = int(got["nitem"][b])
    items = got["items"][b, :nitem]
    expect = set()
    for i, (y0, x0, hy, wx) in enumerate(want.windows):
        for t in range(-(-(hy * wx) // 256)):
            expect.add((i, t))
    assert len(items) == len(expect) and set(map(tuple, items.tolist())) == expect
    # grouped by the parity class of the base window (row and column index of
    # the base tiling); within a class unsplit windows first
    # base windows per row: the oracle's column tiling under the plan's shift
    # (with a shift, two rows may both start at y = 0, so y0 cannot tell rows apart)
    nbx = len(ora.tile_windows(want.Wg, want.w, int(got["shift"][1])))
    parent = want.parent[items[:, 0]]
    cls = ((parent // nbx) % 2) * 2 + (parent % nbx) % 2
    split = want.split[parent].astype(int)
    key = cls * 2 + split
    assert not np.any(np.diff(key) < 0), "items must run class by class, unsplit first"
    for c in range(4):
        assert int(got["nclass"][b, c]) == int(np.sum(cls == c))
    # windows of one class never overlap
    for c in range(4):
        cover = np.zeros((want.Hg, want.Wg), dtype=np.int32)
        for i in sorted(set(items[cls == c, 0].tolist())):
            y0, x0, hy, wx = want.windows[i]
            cover[y0:y0 + hy, x0:x0 + wx] += 1
        assert cover.max() <= 1


@pytest.mark.parametrize("name,step", [(n, s) for n in ALL for s in _steps(n)])
def test_plan_bitexact(name, step):
    cfg = CONFIGS[name]
    src = gr.host_src(name)
    E = ora.dwt_detail(src, cfg.Hg, cfg.Wg)
    w = cfg.schedule[step]
    want = ora.window_plan(E[0], cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
    energy = torch.from_numpy(E).cuda()
    _, plan, _ = gr.gpu_plan(energy, cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
    got = gr.parse(plan)
    gr.compare_plan(got, want)
    Etok = ora.token_energy(E[0]).reshape(-1)
    assert np.array_equal(got["order"][0], ora.global_rank(Etok))
    _check_items(got, want)


@pytest.mark.parametrize("name", ALL)
@pytest.mark.parametrize("seed", [1, 12345, 2 ** 63 + 7])
def test_plan_seeded_bitexact(name, seed):
    # border jitter and random Halo widths drawn from the seed, at every step
    cfg = CONFIGS[name]
    src = gr.host_src(name)
    E = ora.dwt_detail(src, cfg.Hg, cfg.Wg)
    energy = torch.from_numpy(E).cuda()
    for step, w in enumerate(cfg.schedule):
        s = seed + step
        want = ora.window_plan(E[0], cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr, seed=s)
        pcfg = gr.area.make_cfg(cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr, s)
        nbytes = gr.area.area_window_plan_bytes(pcfg)
        plan = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        gr.area.area_window_plan(energy, pcfg, plan, nbytes)
        got = gr.parse(plan)
        assert got["shift"] == ora.jitter_shifts(s, cfg.Hg, cfg.Wg, w)
        gr.compare_plan(got, want)
        _check_items(got, want)


def test_plan_seeded_two_batch_elements():
    rng = np.random.default_rng(5)
    Hg, Wg, w, h, G, seed = 40, 28, 12, 6, 9, 777
    E = (rng.random((2, Hg // 2, Wg // 2)) ** 2).astype(np.float32)
    pcfg = gr.area.make_cfg(2, Hg, Wg, w, h, G, 0.2, seed)
    nbytes = gr.area.area_window_plan_bytes(pcfg)
    plan = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    gr.area.area_window_plan(torch.from_numpy(E).cuda(), pcfg, plan, nbytes)
    got = gr.parse(plan)
    for b in range(2):
        want = ora.window_plan(E[b], Hg, Wg, w, h, G, 0.2, seed=seed, b=b)
        gr.compare_plan(got, want, b)
        _check_items(got, want, b)


@pytest.mark.parametrize("Hg,Wg,w,h,G,thr", [
    (16, 16, 7, 2, 5, 0.3),      # odd window side: unequal quadrants
    (12, 20, 64, 0, 3, 0.0),     # one window covers the grid, no halo
    (10, 14, 4, 1, 0, 9.0),      # G = 0, everything split
    (6, 6, 2, 3, 40, 9.0),       # halo larger than the window, G > N - |ext|
    (34, 18, 9, 1, 7, 0.25),     # ragged tiling
])
def test_plan_edge_cases(Hg, Wg, w, h, G, thr):
    rng = np.random.default_rng(Hg * Wg + w)
    E = (rng.random((2, Hg // 2, Wg // 2)) ** 2).astype(np.float32)
    E[:, :, : max(1, Wg // 4)] = 0.0        # ties at zero energy
    energy = torch.from_numpy(E).cuda()
    _, plan, _ = gr.gpu_plan(energy, 2, Hg, Wg, w, h, G, thr)
    got = gr.parse(plan)
    for b in range(2):
        want = ora.window_plan(E[b], Hg, Wg, w, h, G, thr)
        gr.compare_plan(got, want, b)
        _check_items(got, want, b)


# ---------------------------------------------------------------------------
# Detail map + planner in one cooperative launch: bit-identical to the two
# separate calls (whose output the tests above pin to the oracle)
# ---------------------------------------------------------------------------

def _plan_pair(dsrc, C, dtype, B, Hg, Wg, w, h, G, thr, seed=0, mode=gr.area.AREA_DETAIL_HH):
    pcfg = gr.area.make_cfg(B, Hg, Wg, w, h, G, thr, seed)
    nb = gr.area.area_window_plan_bytes(pcfg)
    p_sep = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    p_fus = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    e_sep = torch.zeros((B, Hg // 2, Wg // 2), dtype=torch.float32, device="cuda")
    e_fus = torch.zeros_like(e_sep)
    gr.area.area_dwt_detail(dsrc, gr.area_dtype(dtype), C, e_sep, B, Hg, Wg, mode)
    gr.area.area_window_plan(e_sep, pcfg, p_sep, nb)
    gr.area.area_dwt_window_plan(dsrc, gr.area_dtype(dtype), C, mode, e_fus, pcfg, p_fus, nb)
    torch.cuda.synchronize()
    assert gr.area.area_kernel_error() == 0
    assert torch.equal(e_fus.view(torch.int32), e_sep.view(torch.int32))
    # header and every section up to the sort scratch, byte for byte
    hdr = p_sep[:256].cpu().numpy().view(np.int64)
    end = int(hdr[10 + gr.area.SECTIONS.index("SCRATCH")])
    assert torch.equal(p_fus[:end], p_sep[:end])
    return e_fus, p_fus


@pytest.mark.parametrize("name", ALL)
def test_fused_dwt_plan_matches_separate_calls(name):
    cfg = CONFIGS[name]
    dsrc = gr.to_dev(gr.host_src(name), cfg.dtype)
    for step in sorted({0, len(cfg.schedule) // 2, len(cfg.schedule) - 1}):
        _plan_pair(dsrc, cfg.C, cfg.dtype, cfg.B, cfg.Hg, cfg.Wg, cfg.schedule[step], cfg.halo,
                   cfg.G, cfg.split_thr)
    # seeded border jitter and Halo widths
    _plan_pair(dsrc, cfg.C, cfg.dtype, cfg.B, cfg.Hg, cfg.Wg, cfg.schedule[-1], cfg.halo, cfg.G,
               cfg.split_thr, seed=99)


@pytest.mark.parametrize("B,C,Hg,Wg,w,h,G,thr,dtype,mode", [
    (2, 16, 40, 28, 12, 6, 9, 0.2, "bf16", 0),     # two batch elements
    (3, 5, 34, 18, 9, 1, 7, 0.25, "fp32", 0),      # odd channel count: scalar loads
    (1, 16, 64, 48, 24, 4, 130, 0.3, "bf16", 1),   # all three detail bands
    (1, 8, 6, 6, 2, 3, 40, 9.0, "fp32", 0),        # halo larger than the window
])
def test_fused_dwt_plan_edge_cases(B, C, Hg, Wg, w, h, G, thr, dtype, mode):
    rng = np.random.default_rng(B * 1000 + Hg)
    src = rng.standard_normal((B, Hg * Wg, C)).astype(np.float32)
    src[:, : Hg * Wg // 3] *= 0.05                 # smooth part: some windows split
    dsrc = gr.to_dev(src, dtype)
    e, plan = _plan_pair(dsrc, C, dtype, B, Hg, Wg, w, h, G, thr, seed=0, mode=mode)
    # and against the oracle directly
    hsrc = gr.to_host(dsrc).astype(np.float32)
    E = ora.dwt_detail(hsrc, Hg, Wg, "hh" if mode == 0 else "all3")
    assert np.array_equal(e.cpu().numpy().view(np.uint32), E.view(np.uint32))
    got = gr.parse(plan)
    for b in range(B):
        want = ora.window_plan(E[b], Hg, Wg, w, h, G, thr)
        gr.compare_plan(got, want, b)
        _check_items(got, want, b)


# ---------------------------------------------------------------------------
# Per-configuration tests (grouped by config: inputs are generated once)
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module", params=ALL)
def data(request):
    d = gr.ConfigData(request.param)
    yield d
    d.release()


def test_pool_kv(data):
    cfg, k, v = data.cfg, data.k, data.v
    heads = [0, cfg.H // 2, cfg.H - 1]
    for mode, mname in [(0, "mean"), (1, "center")]:
        kp, vp = gr.gpu_pool(data.dk, data.dv, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, cfg.f, mode,
                             cfg.dtype)
        for t_dev, t_host in [(kp, k), (vp, v)]:
            got = gr.to_host(t_dev[:, heads])
            want = ora.pool_kv(t_host[:, heads], cfg.Hg, cfg.Wg, cfg.f, mname)
            if cfg.dtype == "bf16":   # one bf16 rounding of the output: 2^-8 relative
                assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) * 1.0001 + 1e-30)
            else:
                gr.assert_close(got, want, "fp32", f"pool {cfg.name} {mname}")


def test_coarse_attn(data):
    cfg, q, k, v = data.cfg, data.q, data.k, data.v
    kp, vp = gr.gpu_pool(data.dk, data.dv, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, cfg.f, 0,
                         cfg.dtype)
    o = gr.gpu_dense(data.dq, kp, vp, cfg.B, cfg.H, cfg.N, cfg.Nk, cfg.D, cfg.scale, cfg.dtype)
    heads = list(range(cfg.H)) if cfg.tiny else [0, 7, cfg.H - 1]
    rows = np.arange(cfg.N) if cfg.tiny else gr.sample_rows(cfg.N, 384, seed=1)
    okp = ora.pool_kv(k[:, heads], cfg.Hg, cfg.Wg, cfg.f)
    ovp = ora.pool_kv(v[:, heads], cfg.Hg, cfg.Wg, cfg.f)
    want = ora.coarse_attn(q[:, heads], okp, ovp, cfg.scale, rows=rows)
    got = gr.to_host(o[:, heads][:, :, torch.from_numpy(rows).cuda()])
    gr.assert_close(got, want, cfg.dtype, f"coarse {cfg.name}")


def test_full_attn(data):
    cfg, q, k, v = data.cfg, data.q, data.k, data.v
    o = torch.empty_like(data.dq)
    gr.area.area_full_attn(data.dq, data.dk, data.dv, o, cfg.B, cfg.H, cfg.N, cfg.D, cfg.scale,
                           gr.area_dtype(cfg.dtype))
    heads = list(range(cfg.H)) if cfg.tiny else [0, cfg.H // 2, cfg.H - 1]
    rows = np.arange(cfg.N) if cfg.tiny else gr.sample_rows(cfg.N, 96, seed=2)
    want = ora.full_attn(q[:, heads], k[:, heads], v[:, heads], cfg.scale, rows=rows)
    got = gr.to_host(o[:, heads][:, :, torch.from_numpy(rows).cuda()])
    gr.assert_close(got, want, cfg.dtype, f"full {cfg.name}")


@pytest.mark.parametrize("step", range(8))
def test_window_attn(data, step):
    cfg = data.cfg
    if step >= len(cfg.schedule):
        pytest.skip("schedule has fewer steps")
    w = cfg.schedule[step]
    energy = gr.gpu_dwt(data.dsrc, cfg.B, cfg.Hg, cfg.Wg, cfg.C, cfg.dtype)
    pcfg, plan, nbytes = gr.gpu_plan(energy, cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G,
                                     cfg.split_thr)
    o = gr.gpu_window(data.dq, data.dk, data.dv, pcfg, plan, nbytes, cfg.H, cfg.D, cfg.scale,
                      cfg.dtype)
    E = ora.dwt_detail(data.src, cfg.Hg, cfg.Wg)
    oplan = ora.window_plan(E[0], cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
    gr.compare_plan(gr.parse(plan), oplan)
    heads = list(range(cfg.H)) if cfg.tiny else [0, cfg.H // 2, cfg.H - 1]
    rows = np.arange(cfg.N) if cfg.tiny else gr.sample_rows(cfg.N, 256, seed=3 + step)
    want = ora.window_attn(data.q, data.k, data.v, [oplan], cfg.scale, rows=rows, heads=heads)
    got = gr.to_host(o[:, heads][:, :, torch.from_numpy(rows).cuda()])
    gr.assert_close(got, want, cfg.dtype, f"window {cfg.name} step {step} w={w}")
    assert gr.area.area_kernel_error() == 0


def test_coarse_attn_ramp_floor(data):
    # Phase I at the floor of the pooling ramp (f = 2): 4x-16x more keys than
    # the configs' fixed factor (16384 keys at 4096^2)
    cfg, q, k, v = data.cfg, data.q, data.k, data.v
    if cfg.f == 2:
        pytest.skip("the config already pools with f = 2")
    f = 2
    Nk = (cfg.Hg // f) * (cfg.Wg // f)
    kp, vp = gr.gpu_pool(data.dk, data.dv, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, f, 0, cfg.dtype)
    o = gr.gpu_dense(data.dq, kp, vp, cfg.B, cfg.H, cfg.N, Nk, cfg.D, cfg.scale, cfg.dtype)
    heads = [0, cfg.H - 1]
    rows = gr.sample_rows(cfg.N, 128, seed=9)
    want = ora.coarse_attn(q[:, heads], ora.pool_kv(k[:, heads], cfg.Hg, cfg.Wg, f),
                           ora.pool_kv(v[:, heads], cfg.Hg, cfg.Wg, f), cfg.scale, rows=rows)
    got = gr.to_host(o[:, heads][:, :, torch.from_numpy(rows).cuda()])
    gr.assert_close(got, want, cfg.dtype, f"coarse f=2 {cfg.name}")


def test_coarse_attn_text(data):
    # Phase I with text tokens: T + N/f^2 keys per query (T ragged: 77)
    cfg, q, k, v = data.cfg, data.q, data.k, data.v
    T = 5 if cfg.tiny else 77
    kt, vt = make_text_kv(cfg, T)
    dkt, dvt = gr.to_dev(kt, cfg.dtype), gr.to_dev(vt, cfg.dtype)
    kp, vp = gr.gpu_pool(data.dk, data.dv, cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D, cfg.f, 0,
                         cfg.dtype)
    o = torch.empty_like(data.dq)
    gr.area.area_coarse_attn_text(data.dq, kp, vp, dkt, dvt, o, cfg.B, cfg.H, cfg.N, cfg.Nk, T,
                                  cfg.D, cfg.scale, gr.area_dtype(cfg.dtype))
    heads = list(range(cfg.H)) if cfg.tiny else [0, cfg.H // 2, cfg.H - 1]
    rows = np.arange(cfg.N) if cfg.tiny else gr.sample_rows(cfg.N, 256, seed=5)
    okp = ora.pool_kv(k[:, heads], cfg.Hg, cfg.Wg, cfg.f)
    ovp = ora.pool_kv(v[:, heads], cfg.Hg, cfg.Wg, cfg.f)
    want = ora.coarse_attn(q[:, heads], okp, ovp, cfg.scale, rows=rows, kt=kt[:, heads],
                           vt=vt[:, heads])
    got = gr.to_host(o[:, heads][:, :, torch.from_numpy(rows).cuda()])
    gr.assert_close(got, want, cfg.dtype, f"coarse+text {cfg.name}")


@pytest.mark.parametrize("which", ["first", "last"])
def test_window_attn_text(data, which):
    cfg = data.cfg
    step = 0 if which == "first" else len(cfg.schedule) - 1
    if cfg.tiny and which == "last":
        pytest.skip("one schedule step")
    T = 5 if cfg.tiny else 77
    kt, vt = make_text_kv(cfg, T)
    dkt, dvt = gr.to_dev(kt, cfg.dtype), gr.to_dev(vt, cfg.dtype)
    w = cfg.schedule[step]
    energy = gr.gpu_dwt(data.dsrc, cfg.B, cfg.Hg, cfg.Wg, cfg.C, cfg.dtype)
    pcfg, plan, nbytes = gr.gpu_plan(energy, cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G,
                                     cfg.split_thr)
    o = torch.empty_like(data.dq)
    wsb = gr.window_ws_bytes(pcfg, cfg.H, cfg.D)
    ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
    gr.area.area_window_attn_text(data.dq, data.dk, data.dv, dkt, dvt, T, pcfg, plan, nbytes, o,
                                  ws, wsb, cfg.H, cfg.D, cfg.scale, gr.area_dtype(cfg.dtype))
    E = ora.dwt_detail(data.src, cfg.Hg, cfg.Wg)
    oplan = ora.window_plan(E[0], cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr)
    heads = list(range(cfg.H)) if cfg.tiny else [0, cfg.H // 2, cfg.H - 1]
    rows = np.arange(cfg.N) if cfg.tiny else gr.sample_rows(cfg.N, 192, seed=11 + step)
    want = ora.window_attn(data.q, data.k, data.v, [oplan], cfg.scale, rows=rows, heads=heads,
                           kt=kt, vt=vt)
    got = gr.to_host(o[:, heads][:, :, torch.from_numpy(rows).cuda()])
    gr.assert_close(got, want, cfg.dtype, f"window+text {cfg.name} step {step}")


@pytest.mark.parametrize("N,Nk,T,D,dtype", [(300, 200, 1, 128, "bf16"), (257, 129, 300, 128, "bf16"),
                                            (130, 70, 33, 64, "fp32"), (100, 64, 128, 64, "bf16")])
def test_dense_attn_text_ragged(N, Nk, T, D, dtype):
    rng = np.random.default_rng(N + T)
    B, H = 2, 2
    q = rng.standard_normal((B, H, N, D)).astype(np.float32)
    k, v = (rng.standard_normal((B, H, Nk, D)).astype(np.float32) for _ in range(2))
    kt, vt = (rng.standard_normal((B, H, T, D)).astype(np.float32) for _ in range(2))
    d = [gr.to_dev(x, dtype) for x in (q, k, v, kt, vt)]
    q, k, v, kt, vt = (gr.to_host(x) for x in d)
    o = torch.empty_like(d[0])
    scale = 1.0 / np.sqrt(D)
    gr.area.area_coarse_attn_text(d[0], d[1], d[2], d[3], d[4], o, B, H, N, Nk, T, D, scale,
                                  gr.area_dtype(dtype))
    gr.assert_close(gr.to_host(o), ora.coarse_attn(q, k, v, scale, kt=kt, vt=vt), dtype,
                    "dense+text")


def test_window_attn_seeded(data):
    # jittered borders and random Halo widths change the plan; the attention
    # kernels consume it unchanged
    cfg = data.cfg
    step = len(cfg.schedule) // 2
    w, seed = cfg.schedule[step], 4242 + step
    energy = gr.gpu_dwt(data.dsrc, cfg.B, cfg.Hg, cfg.Wg, cfg.C, cfg.dtype)
    pcfg = gr.area.make_cfg(cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr, seed)
    nbytes = gr.area.area_window_plan_bytes(pcfg)
    plan = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    gr.area.area_window_plan(energy, pcfg, plan, nbytes)
    o = gr.gpu_window(data.dq, data.dk, data.dv, pcfg, plan, nbytes, cfg.H, cfg.D, cfg.scale,
                      cfg.dtype)
    E = ora.dwt_detail(data.src, cfg.Hg, cfg.Wg)
    oplan = ora.window_plan(E[0], cfg.Hg, cfg.Wg, w, cfg.halo, cfg.G, cfg.split_thr, seed=seed)
    gr.compare_plan(gr.parse(plan), oplan)
    heads = list(range(cfg.H)) if cfg.tiny else [0, cfg.H // 2, cfg.H - 1]
    rows = np.arange(cfg.N) if cfg.tiny else gr.sample_rows(cfg.N, 192, seed=21)
    want = ora.window_attn(data.q, data.k, data.v, [oplan], cfg.scale, rows=rows, heads=heads)
    got = gr.to_host(o[:, heads][:, :, torch.from_numpy(rows).cuda()])
    gr.assert_close(got, want, cfg.dtype, f"window seeded {cfg.name} step {step}")


def _bridge(data, step):
    cfg = data.cfg
    w = cfg.schedule[step]
    ry, rx = gr.area.area_bridge_lattice(w, cfg.Hg, cfg.Wg)
    assert (ry, rx) == ora.bridge_lattice(w, cfg.Hg, cfg.Wg)
    R = ry * rx
    cand = torch.empty((cfg.B, cfg.H, R), dtype=torch.int32, device="cuda")
    wsb = gr.area.area_bridge_select_ws_bytes(cfg.B, cfg.H, cfg.Hg, cfg.Wg, cfg.D)
    ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
    gr.area.area_bridge_select(data.dk, gr.area_dtype(cfg.dtype), cfg.B, cfg.H, cfg.Hg, cfg.Wg,
                               cfg.D, ry, rx, cand, ws, wsb)
    return w, ry, rx, cand


def test_bridge_select_bitexact(data):
    # the pages' rule: per head, most-deviant key per lattice cell
    cfg = data.cfg
    for step in sorted({0, len(cfg.schedule) - 1}):
        w, ry, rx, cand = _bridge(data, step)
        got = cand.cpu().numpy()
        for h in ([0, 1] if cfg.tiny else [0, cfg.H // 2, cfg.H - 1]):
            want = ora.bridge_candidates(data.k[0, h], cfg.Hg, cfg.Wg, ry, rx)
            assert np.array_equal(got[0, h], want), (cfg.name, w, h)


def test_window_attn_bridge(data):
    cfg = data.cfg
    step = len(cfg.schedule) - 1
    w, ry, rx, cand = _bridge(data, step)
    energy = gr.gpu_dwt(data.dsrc, cfg.B, cfg.Hg, cfg.Wg, cfg.C, cfg.dtype)
    pcfg, plan, nbytes = gr.gpu_plan(energy, cfg.B, cfg.Hg, cfg.Wg, w, cfg.halo, 0, cfg.split_thr)
    o = torch.empty_like(data.dq)
    # with the staging area of the candidate rows (bf16: whole tiles as tiles)
    wsb = (gr.area.area_window_attn_ws_bytes(pcfg, cfg.H, cfg.D)
           + gr.area.area_window_attn_bridge_stage_bytes(cfg.B, cfg.H, ry * rx, cfg.D))
    ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
    gr.area.area_window_attn_bridge(data.dq, data.dk, data.dv, cand, ry * rx, pcfg, plan, nbytes,
                                    o, ws, wsb, cfg.H, cfg.D, cfg.scale, gr.area_dtype(cfg.dtype))
    E = ora.dwt_detail(data.src, cfg.Hg, cfg.Wg)
    oplan = ora.window_plan(E[0], cfg.Hg, cfg.Wg, w, cfg.halo, 0, cfg.split_thr)
    heads = list(range(cfg.H)) if cfg.tiny else [0, cfg.H // 2, cfg.H - 1]
    rows = np.arange(cfg.N) if cfg.tiny else gr.sample_rows(cfg.N, 160, seed=31)
    # the oracle's own candidates, from the host keys of the heads under test
    # (the GPU's selection is pinned separately, bit for bit)
    ocand = np.full((cfg.B, cfg.H, ry * rx), -1, dtype=np.int64)
    for h in heads:
        ocand[0, h] = ora.bridge_candidates(data.k[0, h], cfg.Hg, cfg.Wg, ry, rx)
    want = ora.window_attn(data.q, data.k, data.v, [oplan], cfg.scale, rows=rows, heads=heads,
                           bridge=ocand)
    got = gr.to_host(o[:, heads][:, :, torch.from_numpy(rows).cuda()])
    gr.assert_close(got, want, cfg.dtype, f"window bridge {cfg.name} w={w}")


# ---------------------------------------------------------------------------
# Ragged and degenerate shapes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,N,Nk,D,dtype", [
    (1, 1, 1, 1, 128, "bf16"),          # degenerate single query / key
    (2, 3, 1000, 300, 128, "bf16"),     # ragged query and key tails
    (1, 2, 257, 4097, 128, "bf16"),     # key count one past a tile
    (1, 2, 300, 200, 64, "bf16"),       # head_dim 64 on the tensor cores
    (2, 2, 333, 129, 64, "fp32"),
    (1, 2, 130, 70, 128, "fp32"),
])
def test_dense_attn_ragged(B, H, N, Nk, D, dtype):
    rng = np.random.default_rng(N + Nk)
    q = rng.standard_normal((B, H, N, D)).astype(np.float32)
    k = rng.standard_normal((B, H, Nk, D)).astype(np.float32)
    v = rng.standard_normal((B, H, Nk, D)).astype(np.float32)
    dq, dk, dv = gr.to_dev(q, dtype), gr.to_dev(k, dtype), gr.to_dev(v, dtype)
    q, k, v = gr.to_host(dq), gr.to_host(dk), gr.to_host(dv)    # storage-exact values
    scale = 1.0 / np.sqrt(D)
    o = gr.gpu_dense(dq, dk, dv, B, H, N, Nk, D, scale, dtype)
    gr.assert_close(gr.to_host(o), ora.coarse_attn(q, k, v, scale), dtype, "dense ragged")


# ---------------------------------------------------------------------------
# Online softmax: score maxima that grow past the rescale threshold from one
# key tile to the next (O rescaled in TMEM) or fall (the running maximum
# stays ahead of every later tile)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("growing", [True, False])
@pytest.mark.parametrize("D", [128, 64])
def test_dense_attn_rescaled_maxima(growing, D):
    rng = np.random.default_rng(7 + D + growing)
    B, H, N, Nk = 1, 2, 300, 1000
    q = rng.standard_normal((B, H, N, D)).astype(np.float32)
    k = rng.standard_normal((B, H, Nk, D)).astype(np.float32)
    v = rng.standard_normal((B, H, Nk, D)).astype(np.float32)
    # key tile t (128 keys) scaled by 1 + 4t (or the reverse): its row maxima
    # differ from the previous tile's by far more than 2^8 in exp2 units
    t = np.arange(Nk) // 128
    f = 1.0 + 4.0 * (t if growing else t.max() - t)
    k *= f[None, None, :, None].astype(np.float32)
    dq, dk, dv = gr.to_dev(q, "bf16"), gr.to_dev(k, "bf16"), gr.to_dev(v, "bf16")
    q, k, v = gr.to_host(dq), gr.to_host(dk), gr.to_host(dv)
    scale = 1.0 / np.sqrt(D)
    o = gr.gpu_dense(dq, dk, dv, B, H, N, Nk, D, scale, "bf16")
    gr.assert_close(gr.to_host(o), ora.coarse_attn(q, k, v, scale), "bf16", "dense rescaled maxima")


@pytest.mark.parametrize("growing", [True, False])
def test_window_attn_rescaled_maxima(growing):
    rng = np.random.default_rng(11 + growing)
    B, H, Hg, Wg, w, h, G, D = 1, 2, 64, 48, 24, 4, 130, 128
    N = Hg * Wg
    q = rng.standard_normal((B, H, N, D)).astype(np.float32)
    k = rng.standard_normal((B, H, N, D)).astype(np.float32)
    v = rng.standard_normal((B, H, N, D)).astype(np.float32)
    # keys scaled by grid row: the Halo rectangle's 16x8 patches come in row
    # order, so each band of 8 rows raises (or lowers) the row maxima by far
    # more than 2^8 in exp2 units; the global-KV tiles come first
    y = np.arange(N) // Wg
    f = 1.0 + 0.5 * (y if growing else (Hg - 1) - y)
    k *= f[None, None, :, None].astype(np.float32)
    dq, dk, dv = gr.to_dev(q, "bf16"), gr.to_dev(k, "bf16"), gr.to_dev(v, "bf16")
    q, k, v = gr.to_host(dq), gr.to_host(dk), gr.to_host(dv)
    E = (rng.random((B, Hg // 2, Wg // 2)) ** 3).astype(np.float32)
    thr = float(np.median(E))
    pcfg, plan, nbytes = gr.gpu_plan(torch.from_numpy(E).cuda(), B, Hg, Wg, w, h, G, thr)
    scale = 1.0 / np.sqrt(D)
    o = gr.gpu_window(dq, dk, dv, pcfg, plan, nbytes, H, D, scale, "bf16")
    want = ora.window_attn(q, k, v, [ora.window_plan(E[0], Hg, Wg, w, h, G, thr)], scale)
    gr.assert_close(gr.to_host(o), want, "bf16", "window rescaled maxima")


# ---------------------------------------------------------------------------
# Phase II edge cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("Hg,Wg,w,h,G,D,dtype,H", [
    (16, 16, 7, 2, 5, 128, "bf16", 2),     # unequal quadrants, ragged query tiles
    (12, 20, 64, 0, 3, 128, "bf16", 1),    # one window = full attention
    (10, 14, 4, 1, 0, 128, "bf16", 2),     # no global KV
    (24, 40, 12, 3, 17, 64, "bf16", 2),    # head_dim 64 on the tensor cores
    (26, 34, 10, 2, 130, 64, "bf16", 3),   # head_dim 64, global list over two key tiles
    (20, 12, 6, 1, 9, 128, "fp32", 2),     # fp32 head_dim 128
    (64, 48, 24, 4, 130, 128, "bf16", 3),  # global list spans two key tiles
])
def test_window_attn_edge_cases(Hg, Wg, w, h, G, D, dtype, H):
    rng = np.random.default_rng(Hg * 31 + Wg)
    B = 2
    N = Hg * Wg
    q = rng.standard_normal((B, H, N, D)).astype(np.float32)
    k = rng.standard_normal((B, H, N, D)).astype(np.float32)
    v = rng.standard_normal((B, H, N, D)).astype(np.float32)
    dq, dk, dv = gr.to_dev(q, dtype), gr.to_dev(k, dtype), gr.to_dev(v, dtype)
    q, k, v = gr.to_host(dq), gr.to_host(dk), gr.to_host(dv)
    E = (rng.random((B, Hg // 2, Wg // 2)) ** 3).astype(np.float32)
    thr = float(np.median(E))
    pcfg, plan, nbytes = gr.gpu_plan(torch.from_numpy(E).cuda(), B, Hg, Wg, w, h, G, thr)
    scale = 1.0 / np.sqrt(D)
    o = gr.gpu_window(dq, dk, dv, pcfg, plan, nbytes, H, D, scale, dtype)
    plans = [ora.window_plan(E[b], Hg, Wg, w, h, G, thr) for b in range(B)]
    for b in range(B):
        want = ora.window_attn(q[b:b + 1], k[b:b + 1], v[b:b + 1], [plans[b]], scale)
        gr.assert_close(gr.to_host(o[b:b + 1]), want, dtype, "window edge")


@pytest.mark.parametrize("Hg,Wg,w,h,G,D,H", [
    (64, 48, 24, 4, 130, 128, 3),   # one whole staged tile, a gathered partial one
    (64, 64, 24, 4, 512, 128, 2),   # four whole staged tiles
    (26, 34, 10, 2, 256, 64, 3),    # head_dim 64, two whole tiles
    (16, 16, 7, 2, 5, 128, 2),      # no whole tile: nothing staged
])
def test_window_attn_staged_equals_gathered(Hg, Wg, w, h, G, D, H):
    # With room for the staging area the whole global-KV tiles are copied
    # once per call and loaded as tiles; the keys of every tile and their
    # order are the same as when each unit gathers them, so the outputs are
    # identical to the bit.
    rng = np.random.default_rng(Hg * 7 + G)
    B = 2
    N = Hg * Wg
    dq, dk, dv = (gr.to_dev(rng.standard_normal((B, H, N, D)).astype(np.float32), "bf16")
                  for _ in range(3))
    E = (rng.random((B, Hg // 2, Wg // 2)) ** 3).astype(np.float32)
    pcfg, plan, nbytes = gr.gpu_plan(torch.from_numpy(E).cuda(), B, Hg, Wg, w, h, G,
                                     float(np.median(E)))
    scale = 1.0 / np.sqrt(D)
    staged = gr.gpu_window(dq, dk, dv, pcfg, plan, nbytes, H, D, scale, "bf16", staged=True)
    gathered = gr.gpu_window(dq, dk, dv, pcfg, plan, nbytes, H, D, scale, "bf16", staged=False)
    torch.cuda.synchronize()
    assert gr.area.area_window_attn_stage_bytes(pcfg, H, D) > 0
    assert torch.equal(staged, gathered)
    assert gr.area.area_kernel_error() == 0


@pytest.mark.parametrize("Hg,Wg,w,ry,rx,D,H", [
    (64, 64, 16, 16, 16, 128, 2),   # 256 candidates: two whole staged tiles
    (48, 64, 24, 12, 20, 64, 3),    # 240: one whole tile, a gathered partial one
])
def test_window_attn_bridge_staged_equals_gathered(Hg, Wg, w, ry, rx, D, H):
    # the bridged call stages each head's candidate rows of whole tiles when
    # the workspace has room; the outputs are identical to the bit
    rng = np.random.default_rng(Hg + 3 * Wg + D)
    B = 1
    N = Hg * Wg
    dq, dk, dv = (gr.to_dev(rng.standard_normal((B, H, N, D)).astype(np.float32), "bf16")
                  for _ in range(3))
    cand = torch.from_numpy(_gpu_bridge(dk, B, H, Hg, Wg, D, ry, rx, "bf16")).cuda()
    E = (rng.random((B, Hg // 2, Wg // 2)) ** 3).astype(np.float32)
    pcfg, plan, nbytes = gr.gpu_plan(torch.from_numpy(E).cuda(), B, Hg, Wg, w, 2, 0,
                                     float(np.median(E)))
    wmin = gr.area.area_window_attn_ws_bytes(pcfg, H, D)
    outs = []
    for wsb in (wmin + gr.area.area_window_attn_bridge_stage_bytes(B, H, ry * rx, D), wmin):
        o = torch.empty_like(dq)
        ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
        gr.area.area_window_attn_bridge(dq, dk, dv, cand, ry * rx, pcfg, plan, nbytes, o, ws, wsb,
                                        H, D, 1.0 / np.sqrt(D), gr.area.AREA_DTYPE_BF16)
        outs.append(o)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    assert gr.area.area_kernel_error() == 0


@pytest.mark.parametrize("Hg,Wg,w,ry,rx,D,H", [
    (32, 32, 32, 16, 16, 128, 2),   # one window = the grid: every candidate tile masked
    (64, 32, 32, 16, 16, 128, 2),   # two windows: one candidate tile masked, one in part
    (64, 32, 32, 16, 16, 64, 3),    # the same at head_dim 64
])
def test_window_attn_bridge_masked_tiles(Hg, Wg, w, ry, rx, D, H):
    # The candidates come in lattice-cell order, 128 to a tile; a tile whose
    # candidates all lie inside the window's Halo rectangle is masked
    # entirely, so the rows start with a running maximum of -inf and take
    # their first weights from a later tile.
    rng = np.random.default_rng(Hg * 7 + Wg + D)
    B, halo = 1, 2
    N = Hg * Wg
    q, k, v = (rng.standard_normal((B, H, N, D)).astype(np.float32) for _ in range(3))
    dq, dk, dv = gr.to_dev(q, "bf16"), gr.to_dev(k, "bf16"), gr.to_dev(v, "bf16")
    q, k, v = gr.to_host(dq), gr.to_host(dk), gr.to_host(dv)
    cand = torch.from_numpy(_gpu_bridge(dk, B, H, Hg, Wg, D, ry, rx, "bf16")).cuda()
    E = (rng.random((B, Hg // 2, Wg // 2)) ** 3).astype(np.float32)
    thr = 0.0                                  # no window splits
    pcfg, plan, nbytes = gr.gpu_plan(torch.from_numpy(E).cuda(), B, Hg, Wg, w, halo, 0, thr)
    wsb = (gr.area.area_window_attn_ws_bytes(pcfg, H, D)
           + gr.area.area_window_attn_bridge_stage_bytes(B, H, ry * rx, D))
    ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
    o = torch.empty_like(dq)
    scale = 1.0 / np.sqrt(D)
    gr.area.area_window_attn_bridge(dq, dk, dv, cand, ry * rx, pcfg, plan, nbytes, o, ws, wsb,
                                    H, D, scale, gr.area.AREA_DTYPE_BF16)
    oplan = ora.window_plan(E[0], Hg, Wg, w, halo, 0, thr)
    ocand = np.stack([ora.bridge_candidates(k[0, h], Hg, Wg, ry, rx) for h in range(H)])[None]
    want = ora.window_attn(q, k, v, [oplan], scale, bridge=ocand)
    gr.assert_close(gr.to_host(o), want, "bf16", "window bridge, masked candidate tiles")
    assert gr.area.area_kernel_error() == 0


# ---------------------------------------------------------------------------
# the pages' bridge: edge cases of the candidate selection (bit-exact)
# ---------------------------------------------------------------------------

def _gpu_bridge(dk, B, H, Hg, Wg, D, ry, rx, dtype):
    cand = torch.full((B, H, ry * rx), -1, dtype=torch.int32, device="cuda")
    wsb = gr.area.area_bridge_select_ws_bytes(B, H, Hg, Wg, D)
    ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
    gr.area.area_bridge_select(dk, gr.area_dtype(dtype), B, H, Hg, Wg, D, ry, rx, cand, ws, wsb)
    return cand.cpu().numpy()


@pytest.mark.parametrize("B,H,Hg,Wg,ry,rx,D,dtype", [
    (1, 3, 37, 53, 5, 7, 64, "bf16"),      # ragged bands, cells and last chunk
    (2, 1, 33, 64, 33, 64, 128, "bf16"),   # one token per cell
    (1, 2, 40, 41, 3, 2, 128, "fp32"),     # fp32 keys
    (1, 2, 64, 64, 1, 1, 128, "bf16"),     # one cell: the argmax of the whole grid
    (1, 1, 48, 80, 24, 40, 64, "fp32"),    # 2 x 2 cells, fp32 head_dim 64
    (1, 2, 72, 72, 36, 36, 128, "bf16"),   # 2 x 2 cells, band of several tiles
])
def test_bridge_select_edge_cases(B, H, Hg, Wg, ry, rx, D, dtype):
    rng = np.random.default_rng(Hg * 131 + Wg * 7 + D)
    N = Hg * Wg
    k = (rng.standard_normal((B, H, N, D)) * rng.random((B, H, N, 1)) * 3).astype(np.float32)
    dk = gr.to_dev(k, dtype)
    k = gr.to_host(dk)
    got = _gpu_bridge(dk, B, H, Hg, Wg, D, ry, rx, dtype)
    for b in range(B):
        for h in range(H):
            want = ora.bridge_candidates(k[b, h], Hg, Wg, ry, rx)
            assert np.array_equal(got[b, h], want), (b, h)
    if (ry, rx) == (Hg, Wg):
        assert np.array_equal(got[0, 0], np.arange(N))


def test_bridge_select_ties_take_the_first_token():
    # every key equal: all deviations tie, so each cell gives its top-left token
    B, H, Hg, Wg, D, ry, rx = 1, 2, 30, 50, 128, 4, 6
    k = np.full((B, H, Hg * Wg, D), 0.375, dtype=np.float32)
    got = _gpu_bridge(gr.to_dev(k, "bf16"), B, H, Hg, Wg, D, ry, rx, "bf16")
    want = np.array([((cy * Hg) // ry) * Wg + (cx * Wg) // rx
                     for cy in range(ry) for cx in range(rx)], dtype=np.int32)
    for h in range(H):
        assert np.array_equal(got[0, h], want)
        assert np.array_equal(ora.bridge_candidates(k[0, h], Hg, Wg, ry, rx), want)
