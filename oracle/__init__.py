"""fp64 CPU oracle for exact attention.  Test infrastructure only: imported by
the tests, by ``__graft_entry__.smoke()`` and by the CPU-baseline leg of
``bench.py``; never by the product package."""

from .attention import backward, forward, scores

__all__ = ["scores", "forward", "backward"]
