"""CPU oracle for the RainFusion v2 block-sparse attention path (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package; the product path never does.

Modules:
  rainfusion   the path itself: geometry and permutation, block means, ranking
               and selection, float64 attention (any key-block size), E4M3
               quantization of the "mix" precision.
  mxattention  MXFP4 attention: E2M1 rounding with UOS scales, grouped
               quantization of Q, K, V, and the PNQ softmax.
"""
from .rainfusion import *  # noqa: F401,F403
