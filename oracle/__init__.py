"""fp64 CPU oracle for the TurboQuant KV-cache codec.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it. It shares no code, tables or constants with the CUDA
library; it is written from the method's description and pinned by
``tests/test_oracle_*.py`` against closed forms, published values and brute
force.
"""

from .turboquant_oracle import *  # noqa: F401,F403
