"""B200-native 4-bit routed-expert MoE layer (Step-5-Preview shapes).

The compute lives in ``libmoe.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/moe_w4a16.h``).  ``weight_only_bit_route_b200.moe`` is
the thin ctypes binding; importing it loads the library and raises if the
library has not been built.  ``weight_only_bit_route_b200.synthetic`` draws
the seeded synthetic inputs.
"""
__all__ = ["moe", "synthetic"]
