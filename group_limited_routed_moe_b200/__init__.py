"""B200-native group-limited routed MoE layer (Ling-3.0-tiny shapes).

The compute path is the C-ABI library ``libmoe.so`` (hand-written CUDA for
sm_100a); ``group_limited_routed_moe_b200.moe`` is its thin ctypes binding.
Importing this package does not load the library: the binding loads it on
first use and raises if it is missing, so there is no silent fallback.
"""

import importlib

__all__ = ["moe", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
