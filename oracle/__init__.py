"""fp64 CPU oracle of the routed MXFP4 MoE layer (test infrastructure only).

Imported by tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs; never by the product package."""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import mxfp4_pack, mxfp4_values  # noqa: F401
