"""Plain fp64 CPU oracle for cached block attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
leg and its reference arm) may import this package. The CUDA path never does.
"""
from .fbk_oracle import *  # noqa: F401,F403
