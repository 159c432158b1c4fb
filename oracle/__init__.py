"""Float64 CPU oracle of the HGA hot path (test infrastructure only; see hga_oracle)."""
from .hga_oracle import *  # noqa: F401,F403
from .hga_oracle import HGAParams, hga_layer  # noqa: F401
