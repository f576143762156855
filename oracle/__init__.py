"""CPU oracle for the Star Attention hot path -- TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 numpy restatement of what the method computes, written
from the Star Attention pages and checked by the pins in ``tests/`` against
closed forms, library routines and hand-enumerated fixtures.  It shares no code
with the CUDA path and imports nothing from the product package; the product
never imports it.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may call it.

Parity status per function is listed in :mod:`oracle.star_oracle`'s header.
"""

from .star_oracle import *  # noqa: F401,F403
