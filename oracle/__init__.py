"""CPU oracle of the DSA hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The CUDA library does not.
"""
from .dsa_oracle import *  # noqa: F401,F403
