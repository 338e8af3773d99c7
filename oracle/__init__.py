"""CPU oracle of the Sol-Attn hot path (test infrastructure only; see sol_oracle)."""
from .sol_oracle import *  # noqa: F401,F403
from .quant_oracle import *  # noqa: F401,F403
