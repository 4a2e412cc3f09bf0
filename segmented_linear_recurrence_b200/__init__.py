"""librlscan: segmented first-order linear recurrences for RL credit assignment on B200.

The compute lives in the CUDA shared library ``librlscan.so`` (sm_100a),
exposed through the C ABI declared in ``include/rlscan.h``.  This package is
the thin Python binding: ``api`` marshals torch tensors into that ABI and
``synthetic`` draws the seeded benchmark inputs.  Importing the package does
not load the library; the first call does, and raises if it is missing.
"""
from .api import *  # noqa: F401,F403
from .api import __all__  # noqa: F401
