"""fp64 CPU oracle for the Parallax attention forward pass (test infrastructure only)."""
from .plx_oracle import *  # noqa: F401,F403
