"""softmax_ssa_fwd_b200: skip-softmax / N:M sparse flash-attention forward for B200.

The compute path is the C-ABI library ``libssa.so`` (``include/ssa.h``), built
from ``csrc/`` for sm_100a.  ``ssa`` is its thin Python binding (argument
marshalling only); ``inputs`` holds the seeded synthetic workloads.
Importing the binding fails loudly when the library is missing: there is no
fallback.
"""
__all__ = ["ssa", "inputs", "build"]
