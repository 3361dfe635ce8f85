"""Test infrastructure: the float64 CPU oracle of the optimizer step.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.
"""
from .muon_oracle import *  # noqa: F401,F403
