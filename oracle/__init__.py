"""CPU oracle for the RainFusion v2 block-sparse attention path (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package; the product path never does.
"""
from .rainfusion import *  # noqa: F401,F403
