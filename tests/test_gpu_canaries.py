"""Guard bands around every output buffer (a substitute for a memory checker).

Each output is a view into a larger buffer whose leading and trailing bands
hold a byte pattern; after the call the bands must be untouched.  Shapes are
small and ragged (grids and windows that are not tile multiples, clipped
windows, a ragged sort tile), so a write past an edge would land in a band.
"""
import numpy as np
import pytest
import torch

import step_adaptive_sparse_b200 as area

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side of every output
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape` and `dtype` living inside a byte buffer with guards."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(*shape)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.n:]
        return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


def _rand(shape, dtype, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(*shape, generator=g).to(dtype).cuda()


@pytest.mark.parametrize("B,H,Hg,Wg,w,h,G,D,dt", [
    (1, 2, 34, 18, 9, 1, 7, 128, torch.bfloat16),    # ragged tiling, odd window side
    (2, 1, 40, 28, 12, 3, 130, 128, torch.bfloat16),  # global list over two key tiles
    (1, 2, 24, 40, 12, 2, 17, 64, torch.float32),     # CUDA-core path, head_dim 64
    (2, 3, 26, 34, 10, 2, 21, 64, torch.bfloat16),    # tensor cores, head_dim 64, overlaps
])
def test_phase2_outputs_stay_in_bounds(B, H, Hg, Wg, w, h, G, D, dt):
    N = Hg * Wg
    adt = area.AREA_DTYPE_BF16 if dt == torch.bfloat16 else area.AREA_DTYPE_F32
    q, k, v = (_rand((B, H, N, D), dt, s) for s in (1, 2, 3))
    src = _rand((B, N, 16), dt, 4)
    energy = Guarded((B, Hg // 2, Wg // 2), torch.float32)
    area.area_dwt_detail(src, adt, 16, energy.t, B, Hg, Wg, area.AREA_DETAIL_HH)
    assert energy.intact()
    cfg = area.make_cfg(B, Hg, Wg, w, h, G, float(energy.t.mean()))
    nb = area.area_window_plan_bytes(cfg)
    plan = Guarded((nb,), torch.uint8)
    area.area_window_plan(energy.t, cfg, plan.t, nb)
    assert plan.intact()
    plan2 = Guarded((nb,), torch.uint8)
    energy2 = Guarded((B, Hg // 2, Wg // 2), torch.float32)
    area.area_dwt_window_plan(src, adt, 16, area.AREA_DETAIL_HH, energy2.t, cfg, plan2.t, nb)
    assert plan2.intact() and energy2.intact()
    wsb = area.area_window_attn_ws_bytes(cfg, H, D)
    ws = Guarded((wsb // 4,), torch.float32)
    o = Guarded((B, H, N, D), dt)
    area.area_window_attn(q, k, v, cfg, plan.t, nb, o.t, ws.t, wsb, H, D, D ** -0.5, adt)
    assert o.intact() and ws.intact()
    # the same call with the staging area of the global-KV rows: the staging
    # copy and the tiled loads stay inside it, and the output is the same
    wsb2 = wsb + area.area_window_attn_stage_bytes(cfg, H, D)
    ws2 = Guarded((wsb2 // 4,), torch.float32)
    o2 = Guarded((B, H, N, D), dt)
    area.area_window_attn(q, k, v, cfg, plan.t, nb, o2.t, ws2.t, wsb2, H, D, D ** -0.5, adt)
    assert o2.intact() and ws2.intact()
    assert torch.equal(o2.t, o.t)
    assert area.area_kernel_error() == 0


@pytest.mark.parametrize("B,H,Hg,Wg,f,D,dt", [
    (1, 2, 36, 20, 2, 128, torch.bfloat16),
    (2, 1, 30, 18, 3, 128, torch.bfloat16),
    (1, 2, 20, 12, 2, 64, torch.float32),
])
def test_phase1_outputs_stay_in_bounds(B, H, Hg, Wg, f, D, dt):
    N, Nk = Hg * Wg, (Hg // f) * (Wg // f)
    adt = area.AREA_DTYPE_BF16 if dt == torch.bfloat16 else area.AREA_DTYPE_F32
    q, k, v = (_rand((B, H, N, D), dt, s) for s in (5, 6, 7))
    kp, vp = Guarded((B, H, Nk, D), dt), Guarded((B, H, Nk, D), dt)
    area.area_pool_kv(k, v, kp.t, vp.t, B, H, Hg, Wg, D, f, area.AREA_POOL_MEAN, adt)
    assert kp.intact() and vp.intact()
    o = Guarded((B, H, N, D), dt)
    area.area_coarse_attn(q, kp.t, vp.t, o.t, B, H, N, Nk, D, D ** -0.5, adt)
    assert o.intact()
    o2 = Guarded((B, H, N, D), dt)
    area.area_full_attn(q, k, v, o2.t, B, H, N, D, D ** -0.5, adt)
    assert o2.intact()
    assert area.area_kernel_error() == 0


def test_bridge_outputs_stay_in_bounds():
    B, H, Hg, Wg, D, ry, rx = 1, 3, 37, 53, 128, 5, 7
    k = _rand((B, H, Hg * Wg, D), torch.bfloat16, 8)
    cand = Guarded((B, H, ry * rx), torch.int32)
    wsb = area.area_bridge_select_ws_bytes(B, H, Hg, Wg, D)
    ws = Guarded((wsb // 4,), torch.float32)
    area.area_bridge_select(k, area.AREA_DTYPE_BF16, B, H, Hg, Wg, D, ry, rx, cand.t, ws.t, wsb)
    assert cand.intact() and ws.intact()
    assert area.area_kernel_error() == 0


def test_bridged_window_outputs_stay_in_bounds():
    # 16 x 16 = 256 candidates per head: two whole tiles staged per head
    B, H, Hg, Wg, D, ry, rx, w = 1, 2, 40, 56, 128, 16, 16, 12
    N = Hg * Wg
    q, k, v = (_rand((B, H, N, D), torch.bfloat16, s) for s in (9, 10, 11))
    cand = torch.empty((B, H, ry * rx), dtype=torch.int32, device="cuda")
    swsb = area.area_bridge_select_ws_bytes(B, H, Hg, Wg, D)
    sws = torch.empty(swsb // 4, dtype=torch.float32, device="cuda")
    area.area_bridge_select(k, area.AREA_DTYPE_BF16, B, H, Hg, Wg, D, ry, rx, cand, sws, swsb)
    src = _rand((B, N, 16), torch.bfloat16, 12)
    energy = torch.empty((B, Hg // 2, Wg // 2), dtype=torch.float32, device="cuda")
    area.area_dwt_detail(src, area.AREA_DTYPE_BF16, 16, energy, B, Hg, Wg, area.AREA_DETAIL_HH)
    cfg = area.make_cfg(B, Hg, Wg, w, 2, 0, float(energy.mean()))
    nb = area.area_window_plan_bytes(cfg)
    plan = torch.empty(nb, dtype=torch.uint8, device="cuda")
    area.area_window_plan(energy, cfg, plan, nb)
    outs = []
    for extra in (area.area_window_attn_bridge_stage_bytes(B, H, ry * rx, D), 0):
        wsb = area.area_window_attn_ws_bytes(cfg, H, D) + extra
        ws = Guarded((wsb // 4,), torch.float32)
        o = Guarded((B, H, N, D), torch.bfloat16)
        area.area_window_attn_bridge(q, k, v, cand, ry * rx, cfg, plan, nb, o.t, ws.t, wsb, H, D,
                                     D ** -0.5, area.AREA_DTYPE_BF16)
        assert o.intact() and ws.intact()
        outs.append(o.t.clone())
    assert torch.equal(outs[0], outs[1])
    assert area.area_kernel_error() == 0
