"""fp64 CPU oracle of the routed-expert MoE layer (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may use
this package; the product path never imports it.
"""
from .moe_oracle import *  # noqa: F401,F403
