"""CPU oracle for GPTQ's per-layer solve — test infrastructure only (see gptq_oracle)."""
from .gptq_oracle import *  # noqa: F401,F403
from . import gptq_oracle  # noqa: F401
