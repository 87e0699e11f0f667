"""CPU oracle (test infrastructure only; see fva_oracle's header)."""
from .fva_oracle import *  # noqa: F401,F403
from .fva_oracle import __all__  # noqa: F401
