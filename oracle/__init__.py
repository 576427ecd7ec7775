"""CPU oracle (test infrastructure only): see ``oracle.tpa_oracle``."""
from .tpa_oracle import *  # noqa: F401,F403
