"""CPU oracle of the AReA attention hot path -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  The library and its binding never do.
"""
from . import area_oracle  # noqa: F401
