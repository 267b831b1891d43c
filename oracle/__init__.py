"""CPU oracle of the fused MoE FFN layer.  Test infrastructure only (see moe_oracle)."""
from . import moe_oracle  # noqa: F401
