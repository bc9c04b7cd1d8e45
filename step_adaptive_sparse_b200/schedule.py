"""Host-side AReA schedules, marshalled to libarea's host functions.

Pages: ai.info "Methodology in Plain English" (Phase I: the pooling factor
ramps down linearly to f_min = 2, each value snapped to a valid grid divisor;
Phase II: window sides shrink geometrically from w_start to w_min, bridge
R = (rho w)^2 with rho = 0.5; "Scheduling the switch": Phase I ends at a noise
level sigma*), gpt-diffusion.com "Las dos fases de AReA" (the printed ramp
[4,4,4,4,2,2,2,2] at a 256x256 grid).  The arithmetic lives in the library
(area_pool_ramp, area_window_sides, area_bridge_lattice, area_phase_switch,
area_schedule); the kernels never evaluate it.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

from . import binding as _b

PHASE_COARSE = _b.AREA_PHASE_COARSE
PHASE_WINDOW = _b.AREA_PHASE_WINDOW


def pool_ramp(f0: int, f_min: int, steps: int, Hg: int, Wg: int) -> List[int]:
    """Pooling factor per Phase I step (linear f0 -> f_min, nearest common
    divisor of the grid sides, the larger on a tie)."""
    return _b.area_pool_ramp(f0, f_min, steps, Hg, Wg)


def window_schedule(w0: int, w_min: int, steps: int = 8) -> List[int]:
    """Window side per Phase II step:
    w_t = 8 * floor(w0 * (w_min / w0) ** (t / (steps - 1)) / 8 + 1/2), at least 8."""
    return _b.area_window_sides(w0, w_min, steps)


def bridge_lattice(w: int, Hg: int, Wg: int) -> Tuple[int, int]:
    """Cells per axis (ry, rx) of the global-KV bridge for window side w."""
    return _b.area_bridge_lattice(w, Hg, Wg)


def phase_switch(sigmas: Sequence[float], sigma_star: float) -> int:
    """Number of leading steps with sigma >= sigma* (fp32): the Phase I steps."""
    return _b.area_phase_switch(sigmas, sigma_star)


def schedule(sigmas: Sequence[float], sigma_star: float, f0: int, f_min: int, w0: int,
             w_min: int, Hg: int, Wg: int) -> List[Tuple[int, int]]:
    """Per step (PHASE_COARSE, f) or (PHASE_WINDOW, w) for a whole sampling run."""
    return _b.area_schedule(sigmas, sigma_star, f0, f_min, w0, w_min, Hg, Wg)
