"""fp64 CPU oracle (test infrastructure; never imported by the product path)."""
from .psa_oracle import *  # noqa: F401,F403
from .psa_oracle import __all__  # noqa: F401
