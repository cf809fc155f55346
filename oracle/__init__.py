"""Float64 CPU oracle -- test infrastructure only (see svg_oracle)."""
from .svg_oracle import *  # noqa: F401,F403
