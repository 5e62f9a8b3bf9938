"""Float64 CPU oracle of the VDN-H3 hybrid attention layer (test infrastructure only)."""
from . import vdn_oracle  # noqa: F401
