"""fp64 CPU oracle for the Parallax attention forward pass, its gradients and the q/k/v/rho projection (test infrastructure only)."""
from .plx_oracle import *  # noqa: F401,F403
from .plx_oracle_bwd import *  # noqa: F401,F403
from .plx_oracle_stream import *  # noqa: F401,F403
from .plx_oracle_proj import *  # noqa: F401,F403
