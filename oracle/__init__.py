"""fp64 CPU oracle of HTTM's merged global-attention layer (test
infrastructure only; the CUDA library never imports it)."""
from .httm_oracle import *  # noqa: F401,F403
