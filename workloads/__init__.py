"""Workload definitions shared by the tests, the benchmark and the oracle's callers.

This package holds only parameters (the five configurations) and seeded input
generators.  It contains none of the method's arithmetic: neither the oracle
nor the CUDA path is imported here, and neither imports this package.
"""
from .configs import CONFIGS, AreaConfig, get_config  # noqa: F401
from .synth import make_qkv, make_detail_source, make_text_kv, texture_mask  # noqa: F401
