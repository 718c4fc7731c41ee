"""CPU oracle (test infrastructure only): fp64 NumPy definition + pure-Python brute force.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use it;
the library never imports it.
"""
from . import brute, oracle  # noqa: F401
