"""CPU oracle for the top-k MoE FFN layer forward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm, never by the product path.  It is
plain numpy in float64 and shares no code with the CUDA library.
"""
from .moe_oracle import *  # noqa: F401,F403
from . import moe_oracle  # noqa: F401
