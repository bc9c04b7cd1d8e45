"""AReA attention hot path on B200: Python face of the libarea C-ABI.

The compute runs in the CUDA kernels of libarea (step_adaptive_sparse_b200/lib);
this package only marshals arguments (see binding.py).  Build the library with
``python -m step_adaptive_sparse_b200.build``.
"""
from .binding import *  # noqa: F401,F403
from .binding import AreaError, area_plan_cfg, library, make_cfg, parse_plan  # noqa: F401

__all__ = [n for n in dir() if n.startswith("area_") or n.startswith("AREA_")] + [
    "AreaError", "area_plan_cfg", "library", "make_cfg", "parse_plan"]
