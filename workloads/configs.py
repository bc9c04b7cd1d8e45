"""The five synthetic workloads and every parameter the AReA pages leave open.

Sources (AReA: Adaptive Receptive-Field Attention, arXiv 2610.17227, as
summarised on the pages listed in the design notes):

* Phase I pools K/V over f x f token blocks onto a grid near the native 64x64
  (gpt-diffusion.com blog, "Las dos fases de AReA", Fase I; ai.info summary,
  "Methodology in Plain English", Phase I).
* Phase II windows shrink geometrically from w_start (about 70% of the longer
  grid side) to the native size, with a Halo ring, DWT-guided quadrant splits
  and a global-KV bridge (same sections, Fase II / Phase II).

Values the pages leave open are fixed here (one table, read by the tests and
the benchmark, passed as plain arguments to both the oracle and the CUDA path):

* pooling operator: mean (the pages' default is the block centre; centre is a
  second mode);
* halo width h: fixed per config (the pages randomise it up to 8);
* window schedule: explicit integer tables
  w_t = 8 * floor(w0 * (w_min / w0) ** (t / 7) / 8 + 1/2), t = 0..7;
* split threshold on the mean HH detail energy of a window: 0.05 for the tiny
  config (stated with it); for the big configs about the image-wide mean HH
  energy of the synthetic field (0.41 FLUX-shaped, 0.54 Qwen-shaped), i.e. a
  window with less detail than the image average counts as smooth: 0.4 / 0.5;
* global-KV rule: top-G tokens by detail energy outside the halo-extended
  window, ties by token index.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Tuple


@dataclass(frozen=True)
class AreaConfig:
    name: str
    B: int
    H: int
    D: int
    dtype: str            # "fp32" or "bf16": storage and MMA input type
    Hg: int               # token-grid rows
    Wg: int               # token-grid columns
    f: int                # Phase I pooling factor
    schedule: Tuple[int, ...]   # Phase II window sides, one per Phase II step
    halo: int             # Halo width h (tokens)
    G: int                # global-KV tokens per window
    split_thr: float      # split a window when its mean HH energy is below this
    C: int                # channels of the detail source
    texture_frac: float   # fraction of 16x16 token blocks carrying iid texture
    field_grid: int       # side of the coarse N(0,1) grid that is upsampled
    tiny: bool = False    # tiny recipe: noise on the left half, not standardised
    pool_mode: str = "mean"
    seeds: Tuple[int, int, int, int, int] = (0, 1, 2, 3, 4)  # Q, K, V, detail, texture mask

    @property
    def N(self) -> int:
        return self.Hg * self.Wg

    @property
    def Nk(self) -> int:
        return (self.Hg // self.f) * (self.Wg // self.f)

    @property
    def scale(self) -> float:
        return 1.0 / (self.D ** 0.5)


CONFIGS = {
    # Tiny CPU-checkable instance (fp32, D=64, 32x32 grid).
    "tiny": AreaConfig(
        name="tiny", B=1, H=2, D=64, dtype="fp32", Hg=32, Wg=32, f=2,
        schedule=(8,), halo=1, G=16, split_thr=0.05, C=4,
        texture_frac=0.0, field_grid=8, tiny=True),
    # FLUX.1-shaped 2048^2 image: 128x128 tokens.
    "flux2048": AreaConfig(
        name="flux2048", B=1, H=24, D=128, dtype="bf16", Hg=128, Wg=128, f=2,
        schedule=(64, 56, 56, 48, 40, 40, 32, 32), halo=4, G=256,
        split_thr=0.4, C=16, texture_frac=0.30, field_grid=16),
    # FLUX.1-shaped 4096^2: 256x256 tokens.
    "flux4096": AreaConfig(
        name="flux4096", B=1, H=24, D=128, dtype="bf16", Hg=256, Wg=256, f=4,
        schedule=(256, 208, 176, 144, 112, 96, 80, 64), halo=4, G=512,
        split_thr=0.4, C=16, texture_frac=0.30, field_grid=16),
    # FLUX.1-shaped 6144^2: 384x384 tokens.
    "flux6144": AreaConfig(
        name="flux6144", B=1, H=24, D=128, dtype="bf16", Hg=384, Wg=384, f=6,
        schedule=(192, 168, 144, 120, 104, 88, 72, 64), halo=4, G=512,
        split_thr=0.4, C=16, texture_frac=0.30, field_grid=16),
    # Qwen-Image-shaped 6144x2048: 384 rows x 128 columns.
    "qwen6144x2048": AreaConfig(
        name="qwen6144x2048", B=1, H=24, D=128, dtype="bf16", Hg=384, Wg=128, f=4,
        schedule=(272, 224, 176, 144, 120, 96, 80, 64), halo=4, G=256,
        split_thr=0.5, C=16, texture_frac=0.50, field_grid=16),
}


def get_config(name: str) -> AreaConfig:
    try:
        return CONFIGS[name]
    except KeyError as e:
        raise KeyError(f"unknown config {name!r}; known: {sorted(CONFIGS)}") from e
