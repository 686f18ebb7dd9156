"""CPU oracle for the SmoothQuant smoothed W8A8 linear (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package. The product path (``post_quantization_calib_b200``) never does.
"""
from .oracle import *  # noqa: F401,F403
