"""CPU oracle (test infrastructure only): see ``lhcal_oracle``."""
from .lhcal_oracle import *  # noqa: F401,F403
