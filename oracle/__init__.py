"""Float64 CPU oracle for the routed MoE layer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import this package.  It shares no code with the CUDA
library.  Every function is pinned by ``tests/test_oracle_*.py``; no function
here is "parity unpinned".
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import (HIDDEN, INTER, N_EXPERTS, N_GROUPS, KEEP_GROUPS, TOPK,  # noqa: F401
                         N_MOE_LAYERS, RouteResult, PermuteResult)
