"""CPU oracle of the MoE FFN layer forward pass (test infrastructure only)."""
from .moe_oracle import *  # noqa: F401,F403
