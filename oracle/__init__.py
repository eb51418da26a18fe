"""FP64 CPU oracle for the Flux Attention hot path.

Test infrastructure only: imported by the tests, by ``__graft_entry__.smoke()`` and by
the CPU-baseline legs of ``bench.py``; never by the product package.
"""
