"""fp64 CPU oracle for the seven estimators and the generic affine scan -- TEST
INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
leg may import anything from this package.  The product library never does.
"""
from .oracle import (affine_scan, affine_scan_grad, affine_scan_tm, discounted_return, elig_trace, episodic_prefix_sum, gae,  # noqa: F401
                     retrace, run, td_lambda, vtrace)
