"""CPU oracle for the SymNMF clustering hot path -- TEST INFRASTRUCTURE.

A plain, slow, float64 restatement of what the library computes, written from
the pages and pinned by the CPU test suite.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the library never does, and it imports nothing from the library.
"""
from .symnmf import *  # noqa: F401,F403
from .symnmf import PINS  # noqa: F401
