"""fp64 CPU oracle of the block-decode step (test infrastructure only)."""
from .dllm_oracle import *  # noqa: F401,F403
