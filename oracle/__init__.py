"""fp64 CPU oracle for the FlexAttention hot path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``, never by the library.
"""
from .flex_oracle import *  # noqa: F401,F403
from . import flex_oracle  # noqa: F401
