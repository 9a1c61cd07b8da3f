"""CPU oracle (test infrastructure only; see gpt_oracle's header)."""
from .gpt_oracle import *  # noqa: F401,F403
from . import gpt_oracle  # noqa: F401
