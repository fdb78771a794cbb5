"""CPU fp64 oracle of the MoE layer (test infrastructure; never on the product path)."""
from .moe_oracle import *  # noqa: F401,F403
