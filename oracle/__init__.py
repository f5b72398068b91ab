"""The float64 CPU oracle of the POET-X layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / ``--impl reference`` arm, never by the library.  It shares no code with the CUDA
path.  Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
invariants, brute force and the hand-derived fixtures in ``tests/golden/``.
"""
from .poetx_ref import *  # noqa: F401,F403
