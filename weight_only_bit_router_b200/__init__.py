"""B200-native weight-only 4-bit routed-expert MoE layer (W4A16).

The compute path is the sm_100a CUDA library libmoe_w4a16.so (C ABI declared
in include/moe_w4a16.h); this package is its thin Python binding.
"""
from ._binding import *  # noqa: F401,F403
from ._binding import lib, exported_symbols, MoeError, MoeShape, ForwardOpts  # noqa: F401
