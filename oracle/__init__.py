"""fp64 CPU oracle for exact attention.

TEST INFRASTRUCTURE ONLY: used by the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The product path never imports it.
"""
from .attention import backward, backward_head, decode, decode_head, forward, forward_head  # noqa: F401
