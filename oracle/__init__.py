"""fp64 CPU oracle (test infrastructure only; never imported by the product path)."""
from .swiglu_oracle import *  # noqa: F401,F403
from .mhffn_oracle import *  # noqa: F401,F403
