"""CPU oracle for the BATQuant online path — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct reference code (C in ``bat_oracle.c`` plus thin
numpy wrappers). Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it. The product package never imports
it, and it imports nothing from the product package.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, library routines, brute force or values the pages print.
"""
from .oracle import *  # noqa: F401,F403
