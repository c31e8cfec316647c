"""fp64 CPU oracle of the InfLLM-V2 sparse-attention path (test infrastructure only)."""
from .infllm2_oracle import *  # noqa: F401,F403
