"""fp64 CPU oracle for masked grouped-query attention -- test infrastructure.

Imported only by the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py``; never by the product path.
"""
