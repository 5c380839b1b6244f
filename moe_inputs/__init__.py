"""Seeded synthetic inputs for the quantized-expert MoE layer.

This package is shared by the CPU oracle and the CUDA path.  It only *makes
inputs*: hidden states, router weights, the router bias of the skewed
workload, and packed expert weights.  It computes nothing that the layer
computes (no routing, no dequantisation, no FFN, no combine).

Packed expert weights are produced the way the workloads describe them:
fp32 masters of N(0, 0.02) are drawn from a counter-based generator and
encoded with the symmetric block quantiser that fixes the packed format.
That encoder is input preparation: the layer reads packed codes and never
quantises anything.  It is written twice -- numpy here, CUDA in
``csrc/gen_device.cu`` for the multi-GB pools -- using only integer
arithmetic and single correctly rounded fp32 operations, so that both
produce identical bytes (checked by a GPU test).
"""

from .gen import *  # noqa: F401,F403
from .gen import __all__  # noqa: F401
