"""fp64 CPU oracle of the MoE feed-forward layer (test infrastructure only)."""
from .moe_oracle import *  # noqa: F401,F403
