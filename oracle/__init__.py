"""CPU oracle for the fused RMSNorm + BitLinear layer (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg import this package.  The product path never does.
"""
from .oracle import Oracle, load  # noqa: F401
