"""fp64 CPU oracle for the HSA decode step: test infrastructure, not product code.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package.
"""
from . import hsa_oracle  # noqa: F401
