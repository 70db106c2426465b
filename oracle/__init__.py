"""fp64 CPU oracle for CD-RGE on LSTMs (test infrastructure only; see zo_oracle)."""
from .zo_oracle import *  # noqa: F401,F403
