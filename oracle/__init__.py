"""CPU oracle (test infrastructure only; see awq_oracle's header)."""
from .awq_oracle import *  # noqa: F401,F403
from .awq_oracle import __all__  # noqa: F401
