"""Host-side AReA schedules: the Phase I pooling ramp and the Phase II window sides.

Pages: ai.info "Methodology in Plain English" (Phase I: the pooling factor
starts where the pooled grid matches the native one and ramps down linearly
to f_min = 2, each value snapped to a valid grid divisor; Phase II: window
sides shrink geometrically from w_start to w_min); gpt-diffusion.com "Las dos
fases de AReA" (the printed ramp [4,4,4,4,2,2,2,2] at a 256x256 grid).
Integer host arithmetic only; the kernels never evaluate it.
"""
from __future__ import annotations

import math
from typing import List


def pool_ramp(f0: int, f_min: int, steps: int, Hg: int, Wg: int) -> List[int]:
    """Pooling factor per Phase I step.

    The linear value f0 + (f_min - f0) * t / (steps - 1) is snapped to the
    nearest factor dividing both grid sides; a tie goes to the larger factor.
    """
    common = [d for d in range(1, min(Hg, Wg) + 1) if Hg % d == 0 and Wg % d == 0]
    ramp = []
    for t in range(steps):
        frac = t / (steps - 1) if steps > 1 else 0.0
        target = f0 + (f_min - f0) * frac
        best = None
        for d in common:
            if best is None or abs(d - target) < abs(best - target) or (
                    abs(d - target) == abs(best - target) and d > best):
                best = d
        ramp.append(best)
    return ramp


def window_schedule(w0: int, w_min: int, steps: int = 8) -> List[int]:
    """Window side per Phase II step, rounded to multiples of 8:
    w_t = 8 * floor(w0 * (w_min / w0) ** (t / (steps - 1)) / 8 + 1/2)."""
    out = []
    for t in range(steps):
        w = w0 * (w_min / w0) ** (t / (steps - 1) if steps > 1 else 0.0)
        out.append(8 * int(math.floor(w / 8 + 0.5)))
    return out


def bridge_lattice(w: int, Hg: int, Wg: int, rho: float = 0.5):
    """Cells per axis (ry, rx) of the global-KV bridge for window side w: the
    pages' R = (rho * w)^2 tokens per window, rho = 0.5, as round(rho * side)
    per axis of the window clipped to the grid (at least 1, at most the side)."""
    hy, wx = min(w, Hg), min(w, Wg)
    ry = min(Hg, max(1, int(math.floor(rho * hy + 0.5))))
    rx = min(Wg, max(1, int(math.floor(rho * wx + 0.5))))
    return ry, rx
