"""Plain, slow, fp64 CPU oracle for the WorldAttention HKV + HSA attention step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` (its ``cpu_baseline`` and ``--impl reference`` arms) may
import or call anything in this package.  The product path -- the CUDA library
and its Python binding -- never does, and shares no code with it.

Every pinned function is checked in ``tests/test_oracle_*.py`` against things
other than itself (dense attention from a library routine, closed forms,
brute-force subset search, hand-derived fixtures in ``tests/golden/``).
"""
from .hsa import *  # noqa: F401,F403
