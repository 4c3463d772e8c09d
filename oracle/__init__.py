"""CPU oracle for the sparse MoE FFN layer forward and backward (test
infrastructure); the backward is ``oracle.moe_backward``.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
and reference legs may import this package.  The product path (the CUDA
library and its Python binding) never calls it.
"""
from .moe_oracle import *  # noqa: F401,F403
from . import moe_backward  # noqa: F401
