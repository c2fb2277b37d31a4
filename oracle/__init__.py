"""CPU oracle for the 2:4 structured-sparse FP8 GEMM path.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline leg, never by the product path.
"""
from . import sp24_oracle  # noqa: F401
