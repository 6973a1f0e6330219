"""CPU oracle of the MLA layer step (fp64 numpy) and a literal-loop brute force.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline / reference leg of bench.py, never by the library itself.
"""
