"""CPU oracle of the MoE forward pass (test infrastructure only; see moe_oracle)."""
from . import moe_oracle  # noqa: F401
