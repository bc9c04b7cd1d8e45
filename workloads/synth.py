"""Seeded synthetic stand-ins for FLUX.1 / Qwen-Image hidden states.

No dataset, prompt set or model weight is used: the pages measure on real
generations, and these fields only reproduce the token-grid shapes and a
smooth-plus-textured value distribution.

Recipe (all NumPy, ``default_rng(seed)``):

* per channel, a coarse N(0,1) grid of side ``field_grid`` (8 tiny, 16 others)
  is bilinearly upsampled (align-corners) to the Hg x Wg token grid;
* big configs: a random subset of 16x16-token blocks (``texture_frac`` of them,
  chosen by one permutation drawn from the texture-mask seed and shared by all
  four tensors of a config) gets N(0,1) iid noise added; the tensor is then
  standardised to mean 0 / variance 1 and rounded to bf16 (round to nearest
  even);
* tiny config: N(0, 0.3^2) iid noise on grid columns < Wg/2, fp32, not
  standardised.

Everything is returned as float32 NumPy arrays whose values are exactly
representable in the config's storage dtype, so the oracle and the GPU path
read bit-identical inputs.  Layouts: Q/K/V ``[B, H, N, D]`` with token index
``y * Wg + x``; detail source ``[B, N, C]`` channels-last.
"""
from __future__ import annotations

import numpy as np

from .configs import AreaConfig

TEX_BLOCK = 16


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), kept as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = (u >> 16) & np.uint32(1)          # finite inputs: no uint32 overflow
    r += np.uint32(0x7FFF)
    r += u
    r &= np.uint32(0xFFFF0000)
    return r.view(np.float32).reshape(x.shape)


def _interp_matrix(n_out: int, n_in: int) -> np.ndarray:
    """Bilinear (align-corners) interpolation weights, shape [n_out, n_in]."""
    m = np.zeros((n_out, n_in), dtype=np.float64)
    if n_out == 1:
        m[0, 0] = 1.0
        return m
    pos = np.arange(n_out, dtype=np.float64) * (n_in - 1) / (n_out - 1)
    i0 = np.minimum(np.floor(pos).astype(np.int64), n_in - 2)
    fr = pos - i0
    m[np.arange(n_out), i0] = 1.0 - fr
    m[np.arange(n_out), i0 + 1] += fr
    return m


def texture_mask(cfg: AreaConfig) -> np.ndarray:
    """Boolean [Hg, Wg] mask of textured tokens (False everywhere for tiny)."""
    mask = np.zeros((cfg.Hg, cfg.Wg), dtype=bool)
    if cfg.tiny:
        mask[:, : cfg.Wg // 2] = True
        return mask
    by, bx = -(-cfg.Hg // TEX_BLOCK), -(-cfg.Wg // TEX_BLOCK)
    n_blocks = by * bx
    n_tex = int(round(cfg.texture_frac * n_blocks))
    rng = np.random.default_rng(cfg.seeds[4])
    chosen = rng.permutation(n_blocks)[:n_tex]
    for b in chosen:
        y, x = divmod(int(b), bx)
        mask[y * TEX_BLOCK:(y + 1) * TEX_BLOCK, x * TEX_BLOCK:(x + 1) * TEX_BLOCK] = True
    return mask


def _field(cfg: AreaConfig, seed: int, lead: int, ch: int) -> np.ndarray:
    """Smooth field plus texture, shape [lead, Hg, Wg, ch], float32, storage-rounded."""
    rng = np.random.default_rng(seed)
    g = cfg.field_grid
    grid = rng.standard_normal((lead, g, g, ch)).astype(np.float64)
    ry = _interp_matrix(cfg.Hg, g)
    rx = _interp_matrix(cfg.Wg, g).astype(np.float32)
    out = np.empty((lead, cfg.Hg, cfg.Wg, ch), dtype=np.float32)
    for i in range(lead):
        t = np.tensordot(ry, grid[i], axes=([1], [0])).astype(np.float32)   # [Hg, g, ch]
        out[i] = np.matmul(rx[None, :, :], t)                                # [Hg, Wg, ch]
    mask = texture_mask(cfg)
    idx = np.flatnonzero(mask.reshape(-1))
    flat = out.reshape(lead, cfg.N, ch)
    if cfg.tiny:
        flat[:, idx, :] += 0.3 * rng.standard_normal((lead, idx.size, ch), dtype=np.float32)
        return out
    if idx.size:
        flat[:, idx, :] += rng.standard_normal((lead, idx.size, ch), dtype=np.float32)
    flat_all = out.reshape(-1)
    s1 = s2 = 0.0
    step = 1 << 24
    for c0 in range(0, flat_all.size, step):
        chunk = flat_all[c0:c0 + step].astype(np.float64)
        s1 += float(chunk.sum())
        s2 += float(np.dot(chunk, chunk))
    mean = s1 / flat_all.size
    std = float(np.sqrt(s2 / flat_all.size - mean * mean))
    out -= np.float32(mean)
    out *= np.float32(1.0 / std)
    if cfg.dtype == "bf16":
        out = round_to_bf16(out)
    return out


def make_qkv(cfg: AreaConfig):
    """Return (Q, K, V), each float32 [B, H, N, D] with storage-exact values."""
    res = []
    for seed in cfg.seeds[:3]:
        t = _field(cfg, seed, cfg.B * cfg.H, cfg.D)                # [B*H, Hg, Wg, D]
        res.append(t.reshape(cfg.B, cfg.H, cfg.N, cfg.D))
    return tuple(res)


def make_detail_source(cfg: AreaConfig) -> np.ndarray:
    """Detail source, float32 [B, N, C] channels-last, storage-exact."""
    t = _field(cfg, cfg.seeds[3], cfg.B, cfg.C)                    # [B, Hg, Wg, C]
    return t.reshape(cfg.B, cfg.N, cfg.C)


def make_text_kv(cfg: AreaConfig, T: int, seed: int = 5):
    """Synthetic text-token keys and values, float32 [B, H, T, D] each.

    Text tokens have no grid: iid N(0, 1) per element (bf16-rounded for the
    bf16 configs).  They stand in for the prompt tokens of a joint-attention
    transformer; no real prompt is used.
    """
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(2):
        t = rng.standard_normal((cfg.B, cfg.H, T, cfg.D)).astype(np.float32)
        out.append(round_to_bf16(t) if cfg.dtype == "bf16" else t)
    return tuple(out)


def flow_sigmas(steps: int = 28, shift: float = 3.0) -> np.ndarray:
    """Noise levels of a synthetic flow-matching sampler, float32 [steps].

    Stand-in for the sampler that drives the phase switch (the pages name a
    noise level sigma* and 28 steps for FLUX.1, but print no noise schedule):
    times t_i = 1 - i / steps, shifted as sigma = s t / (1 + (s - 1) t).  With
    28 steps and s = 3 the levels cross the pages' sigma* range 0.86..0.96
    near step 8.
    """
    t = 1.0 - np.arange(steps, dtype=np.float64) / steps
    return (shift * t / (1.0 + (shift - 1.0) * t)).astype(np.float32)
