"""fp64 CPU oracle for the Star Attention path (test infrastructure only)."""
from .star_oracle import *  # noqa: F401,F403
