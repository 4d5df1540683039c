"""Plain, slow fp64 CPU oracle for the routed MoE FFN layer over MXFP4 experts.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may.  It shares no code, tables or helpers with the CUDA library.
"""
from .moe_oracle import *  # noqa: F401,F403
