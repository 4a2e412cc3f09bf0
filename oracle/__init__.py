"""fp64 CPU oracle for the seven estimators -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
leg may import anything from this package.  The product library never does.
"""
from .oracle import (discounted_return, elig_trace, episodic_prefix_sum, gae, retrace,  # noqa: F401
                     run, td_lambda, vtrace)
