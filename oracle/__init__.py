"""fp64 CPU oracle for GQLA decode attention.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import it.
"""
