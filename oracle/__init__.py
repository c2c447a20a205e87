"""fp64 CPU oracle of the hybrid compressed attention layer (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline /
reference arm use this package.  The CUDA library never imports or calls it.
"""
from .hyb_oracle import *  # noqa: F401,F403
