"""CPU oracle of the W4A16 routed-expert MoE layer: test infrastructure only.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import anything under ``oracle/``.  The CUDA library and its
Python binding never do, and the oracle imports nothing from them.
"""
from .moe_oracle import *  # noqa: F401,F403
