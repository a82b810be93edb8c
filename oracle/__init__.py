"""CPU oracle (test infrastructure only; see krea2_oracle's header)."""
from .krea2_oracle import *  # noqa: F401,F403
