"""fp64 CPU oracle for paged decode attention.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU baseline leg of ``bench.py``.  The CUDA library never uses it.
"""
