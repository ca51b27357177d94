"""Float64 CPU oracle for the HSTU layer forward and backward (TEST INFRASTRUCTURE ONLY).

Only tests, the entry-point smoke check and the benchmark's CPU baseline leg
may import this package.  It shares no code with the CUDA library and never
consumes a value produced by it.
"""
from . import brute, hstu, hstu_bwd  # noqa: F401
