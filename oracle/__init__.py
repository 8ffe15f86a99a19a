"""CPU oracle for the TurboQuant-style KV-cache path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call, link or
execute anything under ``oracle/``; only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline leg (and its ``--impl reference`` arm) use it.
It shares no code with the CUDA library: only the seeded input generators in
``synth`` serve both sides.

See ``oracle/tq_oracle.py`` for the definitions and the passages they follow.
"""
from .tq_oracle import *  # noqa: F401,F403
