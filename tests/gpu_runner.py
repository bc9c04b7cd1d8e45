"""Helpers of the GPU parity tests: run the CUDA path through the C-ABI binding.

Inputs come from the seeded generators of ``workloads``; expected values come
from the oracle.  Nothing here computes any part of the method.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

import step_adaptive_sparse_b200 as area
from workloads import CONFIGS, make_detail_source, make_qkv

TOL = {"bf16": (2e-2, 2e-3), "fp32": (1e-4, 1e-5)}   # (max-abs, mean-abs)


def torch_dtype(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def area_dtype(name):
    return area.AREA_DTYPE_BF16 if name == "bf16" else area.AREA_DTYPE_F32


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(torch_dtype(dtype))


def to_host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


@functools.lru_cache(maxsize=8)
def host_src(name: str) -> np.ndarray:
    return make_detail_source(CONFIGS[name])


@functools.lru_cache(maxsize=1)
def host_qkv(name: str):
    return make_qkv(CONFIGS[name])


class ConfigData:
    """Host (storage-exact float32) and device copies of one config's inputs."""

    def __init__(self, name: str):
        cfg = CONFIGS[name]
        self.name, self.cfg = name, cfg
        self.q, self.k, self.v = host_qkv(name)
        self.src = host_src(name)
        self.dq, self.dk, self.dv = (to_dev(x, cfg.dtype) for x in (self.q, self.k, self.v))
        self.dsrc = to_dev(self.src, cfg.dtype)

    def release(self):
        del self.dq, self.dk, self.dv, self.dsrc
        torch.cuda.empty_cache()


def assert_close(got: np.ndarray, want: np.ndarray, dtype: str, what: str = ""):
    max_tol, mean_tol = TOL[dtype]
    err = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(want, dtype=np.float64))
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= max_tol, f"{what}: max-abs {err.max():.3e} > {max_tol}"
    assert err.mean() <= mean_tol, f"{what}: mean-abs {err.mean():.3e} > {mean_tol}"
    return float(err.max()), float(err.mean())


def sample_rows(N: int, n: int, seed: int = 0) -> np.ndarray:
    """Sorted sample of token rows that always includes the first and last token."""
    rng = np.random.default_rng(seed)
    n = min(n, N)
    rows = set(rng.choice(N, size=n, replace=False).tolist())
    rows.update([0, N - 1])
    return np.array(sorted(rows), dtype=np.int64)


# ---- GPU calls -----------------------------------------------------------------

def gpu_pool(k, v, B, H, Hg, Wg, D, f, mode, dtype):
    Np = (Hg // f) * (Wg // f)
    kp = torch.empty((B, H, Np, D), dtype=k.dtype, device="cuda")
    vp = torch.empty_like(kp)
    area.area_pool_kv(k, v, kp, vp, B, H, Hg, Wg, D, f, mode, area_dtype(dtype))
    return kp, vp


def gpu_dense(q, k, v, B, H, N, Nk, D, scale, dtype):
    o = torch.empty((B, H, N, D), dtype=q.dtype, device="cuda")
    area.area_coarse_attn(q, k, v, o, B, H, N, Nk, D, scale, area_dtype(dtype))
    return o


def gpu_dwt(src, B, Hg, Wg, C, dtype, mode=area.AREA_DETAIL_HH):
    e = torch.empty((B, Hg // 2, Wg // 2), dtype=torch.float32, device="cuda")
    area.area_dwt_detail(src, area_dtype(dtype), C, e, B, Hg, Wg, mode)
    return e


def gpu_plan(energy, B, Hg, Wg, w, halo, G, thr):
    cfg = area.make_cfg(B, Hg, Wg, w, halo, G, thr)
    nbytes = area.area_window_plan_bytes(cfg)
    plan = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    area.area_window_plan(energy, cfg, plan, nbytes)
    return cfg, plan, nbytes


def window_ws_bytes(cfg, H, D, staged=True):
    """Workspace bytes of a window call: the minimum, plus the staging area of
    the global-KV rows (the bf16 fast path) when `staged`."""
    wsb = area.area_window_attn_ws_bytes(cfg, H, D)
    return wsb + area.area_window_attn_stage_bytes(cfg, H, D) if staged else wsb


def gpu_window(q, k, v, cfg, plan, nbytes, H, D, scale, dtype, staged=True):
    o = torch.empty_like(q)
    wsb = window_ws_bytes(cfg, H, D, staged)
    ws = torch.empty(wsb // 4, dtype=torch.float32, device="cuda")
    area.area_window_attn(q, k, v, cfg, plan, nbytes, o, ws, wsb, H, D, scale, area_dtype(dtype))
    return o


def parse(plan: torch.Tensor) -> dict:
    torch.cuda.synchronize()
    return area.parse_plan(plan.cpu().numpy())


def compare_plan(got: dict, want, b: int = 0):
    """Bit-exact comparison of a device plan with an oracle Plan."""
    nb = want.base.shape[0]
    nw = want.windows.shape[0]
    assert got["nb"] == nb
    assert np.array_equal(got["base"][b], want.base)
    assert np.array_equal(got["score"][b].view(np.uint32), want.score.view(np.uint32))
    assert np.array_equal(got["split"][b], want.split)
    assert int(got["nwin"][b]) == nw
    assert np.array_equal(got["win"][b, :nw], want.windows)
    assert np.array_equal(got["parent"][b, :nw], want.parent)
    assert np.array_equal(got["ext"][b, :nw], want.ext)
    assert np.array_equal(got["gcount"][b, :nw], want.gcount)
    if want.G:
        assert np.array_equal(got["gidx"][b, :nw], want.gidx)
    assert np.array_equal(got["wsum"][b].view(np.uint32), want.wsum.view(np.uint32))
    cover = np.zeros((want.Hg, want.Wg), dtype=np.int32)
    for (y0, x0, hy, wx) in want.windows:
        cover[y0:y0 + hy, x0:x0 + wx] += 1
    assert np.array_equal(got["cover"][b], cover.reshape(-1))
