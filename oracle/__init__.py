"""fp64 CPU oracle for ResidualQuant decode attention -- test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.
"""
