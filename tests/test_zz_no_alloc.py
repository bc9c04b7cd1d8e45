"""area_window_attn_noalloc: windowed attention for callers that cannot allocate.

Some callers of this library run where they may not allocate device memory:
inside a host runtime that owns every allocation and hands out only fixed
input and output buffers, or in a serving loop that must not allocate once it
is running.  For them the library offers area_window_attn_noalloc, which takes
no workspace argument and uses a 32 MiB static device array of the library
instead.  These tests check, through the C ABI, that it returns what
area_window_attn returns on two calls in a row (the second call must not see
the first call's leftovers), and that sizes beyond the static array are
refused before anything runs.
"""
import numpy as np
import pytest
import torch

import step_adaptive_sparse_b200 as area

TOL = {area.AREA_DTYPE_BF16: (2e-2, 2e-3), area.AREA_DTYPE_F32: (1e-4, 1e-5)}


def _setup(Hg, Wg, H, D, w, h, G, dtype, seed):
    rng = np.random.default_rng(seed)
    tdt = torch.bfloat16 if dtype == area.AREA_DTYPE_BF16 else torch.float32
    N = Hg * Wg
    qkv = [torch.from_numpy(rng.standard_normal((1, H, N, D)).astype(np.float32)).cuda().to(tdt)
           for _ in range(3)]
    E = (rng.random((1, Hg // 2, Wg // 2)) ** 2).astype(np.float32)
    energy = torch.from_numpy(E).cuda()
    cfg = area.make_cfg(1, Hg, Wg, w, h, G, float(np.median(E)))
    nbytes = area.area_window_plan_bytes(cfg)
    plan = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    area.area_window_plan(energy, cfg, plan, nbytes)
    return qkv, cfg, plan, nbytes


def _with_workspace(q, k, v, cfg, plan, nbytes, H, D, dtype):
    o = torch.empty_like(q)
    wsb = area.area_window_attn_ws_bytes(cfg, H, D)
    ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
    area.area_window_attn(q, k, v, cfg, plan, nbytes, o, ws, wsb, H, D, 1.0 / np.sqrt(D), dtype)
    return o


def _close(a, b, dtype):
    err = (a.float() - b.float()).abs()
    max_tol, mean_tol = TOL[dtype]
    assert torch.isfinite(a.float()).all()
    assert err.max().item() <= max_tol and err.mean().item() <= mean_tol


@pytest.mark.gpu
@pytest.mark.parametrize("Hg,Wg,H,D,w,h,G,dtype", [
    (32, 32, 2, 64, 10, 1, 16, area.AREA_DTYPE_F32),     # CUDA-core path, overlapping windows
    (64, 64, 4, 128, 24, 4, 70, area.AREA_DTYPE_BF16),   # tensor-core path, overlapping windows
])
def test_noalloc_matches_window_attn_on_two_calls(Hg, Wg, H, D, w, h, G, dtype):
    scale = 1.0 / np.sqrt(D)
    for call, seed in enumerate((11, 12)):       # two calls in a row, different inputs
        (q, k, v), cfg, plan, nbytes = _setup(Hg, Wg, H, D, w, h, G, dtype, seed)
        want = _with_workspace(q, k, v, cfg, plan, nbytes, H, D, dtype)
        got = torch.empty_like(q)
        area.area_window_attn_noalloc(q, k, v, cfg, plan, nbytes, got, H, D, scale, dtype)
        torch.cuda.synchronize()
        _close(got, want, dtype)
    assert area.area_kernel_error() == 0


def test_noalloc_refuses_sizes_beyond_the_static_workspace():
    # 48-token windows on a 128x128 grid overlap on 3840 tokens; 24 heads at
    # D = 128 need 3840 * 24 * 128 * 4 bytes = 45 MiB of accumulator rows,
    # more than the 32 MiB array: refused on the host, before any device work
    # (the pointers are never touched).
    cfg = area.make_cfg(1, 128, 128, 48, 4, 256, 0.4)
    assert area.area_window_attn_ws_bytes(cfg, 24, 128) > 32 << 20
    nbytes = area.area_window_plan_bytes(cfg)
    fake = 1 << 20
    with pytest.raises(area.AreaError) as e:
        area.area_window_attn_noalloc(fake, fake, fake, cfg, fake, nbytes, fake, 24, 128,
                                      0.088, area.AREA_DTYPE_BF16)
    assert e.value.status == area.AREA_ENOSPACE
