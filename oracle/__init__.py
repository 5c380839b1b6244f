"""CPU oracle of the routed, quantized-expert MoE FFN layer (test infrastructure).

This package is the correctness reference and nothing else.  Only the test
suite, the smoke check of ``__graft_entry__`` and the CPU-baseline leg of
``bench.py`` may import it; the CUDA library never calls it and shares no code
with it (the one shared module is the seeded input generator ``moe_inputs``).

Everything is evaluated in numpy float64 from the plain definitions, one token
at a time.  See ``moe_oracle`` for the functions and what pins each of them.
"""

from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import __all__  # noqa: F401
