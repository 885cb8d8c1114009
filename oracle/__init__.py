"""CPU oracle for Sol-Attn (test infrastructure only; never on the product path)."""
from .solattn_oracle import *  # noqa: F401,F403
