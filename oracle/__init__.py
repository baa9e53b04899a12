"""CPU oracle of the sparse MoE FFN forward (test infrastructure only; see moe_oracle)."""
from . import moe_oracle  # noqa: F401
