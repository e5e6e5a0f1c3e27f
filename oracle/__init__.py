"""CPU float64 oracle for the DSA forward path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.
"""
from . import dsa_ref  # noqa: F401
