"""CPU oracle for CRISP sparse prefill (test infrastructure only; see crisp_oracle)."""
from .crisp_oracle import *  # noqa: F401,F403
