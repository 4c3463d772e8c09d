"""CPU oracle for the sparse MoE FFN layer forward (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
and reference legs may import this package.  The product path (the CUDA
library and its Python binding) never calls it.
"""
from .moe_oracle import *  # noqa: F401,F403
