"""CPU fp64 oracle for MLA decode (test infrastructure; see ``mla_oracle``)."""
from .mla_oracle import *  # noqa: F401,F403
from .mla_oracle import __all__  # noqa: F401
