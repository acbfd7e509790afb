"""Float64 CPU oracle for RACE attention (test infrastructure, not product code).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.
"""
from .race_oracle import *  # noqa: F401,F403
from . import race_oracle  # noqa: F401
