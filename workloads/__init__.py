"""Workload definitions shared by the tests, the benchmark and the oracle's callers.

This package holds only parameters (the five configurations) and seeded input
generators.  It contains none of the method's arithmetic: neither the oracle
nor the CUDA path is imported here, and neither imports this package.
"""
from .configs import CONFIGS, AreaConfig, get_config  # noqa: F401
from .synth import (flow_sigmas, make_detail_source, make_qkv, make_text_kv,  # noqa: F401
                    texture_mask)
