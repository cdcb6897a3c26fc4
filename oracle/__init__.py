"""fp64 CPU oracle of the ISPA hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does.
"""
from . import ispa_oracle  # noqa: F401
