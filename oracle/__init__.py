"""fp64 CPU oracle of the quantized MoE expert layer (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package. The CUDA library never does.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import LUT_OFFSET  # noqa: F401
