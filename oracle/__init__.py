"""CPU fp64 oracle for the GDLA forward pass (test infrastructure; never on the product path)."""
from .gdla_oracle import *  # noqa: F401,F403
