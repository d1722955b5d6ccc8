"""fp64 CPU oracle of the gated-retention mixer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The GPU library never does.
"""
from .gret_oracle import *  # noqa: F401,F403
