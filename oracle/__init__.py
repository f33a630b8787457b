"""Float64 CPU oracle (test infrastructure; never used by the product path)."""
from .wf_oracle import *  # noqa: F401,F403
