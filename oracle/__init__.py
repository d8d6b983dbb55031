"""fp64 CPU oracle of the LCSA hot path.

Test infrastructure only: used by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference arm of ``bench.py``; never by the product path.
"""
