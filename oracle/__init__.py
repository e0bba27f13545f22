"""CPU oracle for the fine-grained MoE FFN layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm
may import this package. The product path (the CUDA library and its binding) never does.
"""
from .moe_oracle import *  # noqa: F401,F403
