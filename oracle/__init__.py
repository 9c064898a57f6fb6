"""fp64 CPU oracle for exact attention.  Test infrastructure only: imported by
the tests, by ``__graft_entry__.smoke()`` and by the CPU-baseline leg of
``bench.py``; never by the product package."""

from .attention import backward, forward, scores
from .fp8 import e4m3_decode, forward_fp8

__all__ = ["scores", "forward", "backward", "e4m3_decode", "forward_fp8"]
