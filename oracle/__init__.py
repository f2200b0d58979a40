"""fp64 CPU oracle for ReHyAt's chunked hybrid attention.

Test infrastructure: imported only by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The product path never uses it.
"""
from .rehyat_oracle import *  # noqa: F401,F403
